// decompress.cu -- W = the rebuilt weights, written out in fp32.
//
// Eq (1) of the paperhub.cn review thread, W_blk = U t, applied to every
// block.  A lane takes 4 consecutive blocks of a row (one 16-byte record
// load) and rebuilds their weights exactly (see seedlm_device.cuh); a warp's
// 32 lanes cover 128 consecutive blocks, staged in shared memory and written
// out with fully coalesced 16-byte streaming stores.  The kernel is bound by
// the 4 bytes per weight it writes, eight times the 0.5 bytes per weight it
// reads.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

SEEDLM_CHECK_FLAG(decompress)

namespace {

constexpr int kThreads = 256;
constexpr int kRecs = 4;  // records per thread per step: one 16-byte load

// The records and exponents of one chunk: 4 consecutive blocks of a row.
struct Chunk {
  uint4 rec;
  uint32_t e;  // C = 12: exponent nibbles of the 4 blocks in bits [0,16)
};

template <int C>
__device__ __forceinline__ Chunk load_chunk(const uint32_t* __restrict__ rec,
                                            const uint8_t* __restrict__ eplane, int rows,
                                            int rec_pitch, int e_pitch, int r, int k) {
  Chunk ch{};
  // The chunk's last record word, and its exponent bytes, lie inside row r.
  if (SEEDLM_IN_BOUNDS(g_check_flag, r, rows) &&
      SEEDLM_IN_BOUNDS(g_check_flag, kRecs * k + kRecs - 1, rec_pitch))
    ch.rec = ld_stream_u4(rec + (size_t)r * rec_pitch + kRecs * k);
  ch.e = 0;
  if constexpr (C == 12) {
    const uint8_t* ep = eplane + (size_t)r * e_pitch + 2 * k;
    uint32_t lo = 2 * k < e_pitch ? ld_stream_u8(ep) : 0u;
    uint32_t hi = 2 * k + 1 < e_pitch ? ld_stream_u8(ep + 1) : 0u;
    ch.e = lo | (hi << 8);
  }
  return ch;
}

template <int C>
__device__ __forceinline__ void rebuild_block(uint32_t word, uint32_t e4, const uint32_t* t32,
                                              const uint2* t64, float (&w)[C]) {
  if constexpr (C == 8) {
    const BlockC8 blk = decode_c8(word, t32, t32 + 256);
    const float nm = __uint_as_float(blk.negm);
    w[0] = __int_as_float(weight_bits_c8<0>(blk)) + nm;
    w[1] = __int_as_float(weight_bits_c8<1>(blk)) + nm;
    w[2] = __int_as_float(weight_bits_c8<2>(blk)) + nm;
    w[3] = __int_as_float(weight_bits_c8<3>(blk)) + nm;
    w[4] = __int_as_float(weight_bits_c8<4>(blk)) + nm;
    w[5] = __int_as_float(weight_bits_c8<5>(blk)) + nm;
    w[6] = __int_as_float(weight_bits_c8<6>(blk)) + nm;
    w[7] = __int_as_float(weight_bits_c8<7>(blk)) + nm;
  } else {
    const BlockC12 blk = decode_c12(word, e4, t64, t64 + 256);
    const float nm = __uint_as_float(blk.negm);
    w[0] = __int_as_float(weight_bits_c12<0>(blk)) + nm;
    w[1] = __int_as_float(weight_bits_c12<1>(blk)) + nm;
    w[2] = __int_as_float(weight_bits_c12<2>(blk)) + nm;
    w[3] = __int_as_float(weight_bits_c12<3>(blk)) + nm;
    w[4] = __int_as_float(weight_bits_c12<4>(blk)) + nm;
    w[5] = __int_as_float(weight_bits_c12<5>(blk)) + nm;
    w[6] = __int_as_float(weight_bits_c12<6>(blk)) + nm;
    w[7] = __int_as_float(weight_bits_c12<7>(blk)) + nm;
    w[8] = __int_as_float(weight_bits_c12<8>(blk)) + nm;
    w[9] = __int_as_float(weight_bits_c12<9>(blk)) + nm;
    w[10] = __int_as_float(weight_bits_c12<10>(blk)) + nm;
    w[11] = __int_as_float(weight_bits_c12<11>(blk)) + nm;
  }
}

// A warp item is 32 consecutive chunks (4 blocks each) of one row: lane l
// rebuilds chunk 32j + l into its slice of a per-warp staging buffer (one
// padding float4 per lane keeps the writes conflict-free).  Float4 f of the
// item belongs to column 128 j C + 4 f, so the warp then writes the item
// back with store instructions that each cover 512 contiguous bytes.  The
// next item's records are loaded before the current one is rebuilt.
template <int C>
__global__ void __launch_bounds__(kThreads)
decompress_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane, int rows,
                  int cols, int nb, int rec_pitch, int e_pitch, float* __restrict__ W, int64_t ldw,
                  int vec) {
  constexpr int F = C;  // float4 per chunk (4 blocks x C floats / 4)
  extern __shared__ __align__(16) unsigned char dsm[];
  uint32_t* t32 = reinterpret_cast<uint32_t*>(dsm);
  uint2* t64 = reinterpret_cast<uint2*>(dsm);
  for (int i = threadIdx.x; i < 512; i += kThreads) {
    uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
    if constexpr (C == 8)
      t32[i] = (uint32_t)v;
    else
      t64[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float4* stage = reinterpret_cast<float4*>(dsm + 512 * 8) + warp * 32 * (F + 1);
  // float4 slots of this warp's staging buffer that the launch provides.
  SEEDLM_CHECK_ONLY(const int stage_slots =
                        (int)(seedlm_dynamic_smem_bytes() - 512 * 8) / 16 - warp * 32 * (F + 1);)
  const int cpr = (nb + kRecs - 1) / kRecs;  // chunks per row
  const int ipr = (cpr + 31) / 32;           // warp items per row
  const int64_t items = (int64_t)rows * ipr;
  const int64_t wstep = (int64_t)gridDim.x * (kThreads / 32);
  int64_t it = (int64_t)blockIdx.x * (kThreads / 32) + warp;
  if (it >= items) return;
  auto locate = [&](int64_t item, int& r, int& k) {
    r = (int)(item / ipr);
    k = (int)(item - (int64_t)r * ipr) * 32 + lane;
  };
  int r, k;
  locate(it, r, k);
  Chunk cur = k < cpr ? load_chunk<C>(rec, eplane, rows, rec_pitch, e_pitch, r, k) : Chunk{};
  while (true) {
    const int64_t inext = it + wstep;
    int rn = 0, kn = 0;
    Chunk nxt{};
    if (inext < items) {
      locate(inext, rn, kn);
      if (kn < cpr) nxt = load_chunk<C>(rec, eplane, rows, rec_pitch, e_pitch, rn, kn);
    }
    const uint32_t words[kRecs] = {cur.rec.x, cur.rec.y, cur.rec.z, cur.rec.w};
#pragma unroll
    for (int q = 0; q < kRecs; ++q) {
      float w[C];
      rebuild_block<C>(words[q], (cur.e >> (4 * q)) & 15u, t32, t64, w);
#pragma unroll
      for (int v = 0; v < C / 4; ++v) {
        const int si = lane * (F + 1) + q * (C / 4) + v;
        if (SEEDLM_IN_BOUNDS(g_check_flag, si, stage_slots))
          stage[si] = make_float4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
      }
    }
    __syncwarp();
    const int j = (k - lane) / 32;  // item index within the row
    float* dst_row = W + (size_t)r * (size_t)ldw + (size_t)128 * j * C;
    const int col0 = 128 * j * C;
    // Elements of W the call covers: rows - 1 full pitches plus one row.
    SEEDLM_CHECK_ONLY(const size_t w_extent = (size_t)(rows - 1) * (size_t)ldw + (size_t)cols;
                      const size_t row_base = (size_t)r * (size_t)ldw + (size_t)col0;)
#pragma unroll
    for (int q = 0; q < F; ++q) {
      const int ff = q * 32 + lane;
      const int c = ff / F, v = ff - c * F;
      const float4 val = stage[c * (F + 1) + v];
      const int j0 = col0 + 4 * ff;
      if (vec && j0 + 4 <= cols) {
        if (SEEDLM_IN_BOUNDS(g_check_flag, row_base + 4 * ff + 3, w_extent))
          __stcs(reinterpret_cast<float4*>(dst_row + 4 * ff), val);
      } else if (j0 < cols) {
        const float e4[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (j0 + u < cols && SEEDLM_IN_BOUNDS(g_check_flag, row_base + 4 * ff + u, w_extent))
            dst_row[4 * ff + u] = e4[u];
      }
    }
    __syncwarp();
    if (inext >= items) return;
    it = inext;
    r = rn;
    k = kn;
    cur = nxt;
  }
}

}  // namespace

int launch_decompress(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane, float* W,
                      int64_t ldw, cudaStream_t stream, const DeviceInfo& dev) {
  const int cpr = (f.nb + kRecs - 1) / kRecs;
  const int64_t items = (int64_t)f.rows * ((cpr + 31) / 32);
  if (items == 0) return SEEDLM_OK;
  const int vec = ((reinterpret_cast<uintptr_t>(W) & 15u) == 0 && (ldw % 4) == 0) ? 1 : 0;
  const int warps = kThreads / 32;
  int64_t want = (items + warps - 1) / warps;
  int64_t cap = (int64_t)dev.num_sms * 4;
  int grid = (int)(want < cap ? want : cap);
  const size_t smem = 512 * 8 + (size_t)warps * 32 * (f.C + 1) * 16;
  if (f.C == 8) {
    int rc = allow_max_smem((const void*)decompress_kernel<8>, dev);
    if (rc) return rc;
    decompress_kernel<8><<<grid, kThreads, smem, stream>>>(rec, eplane, f.rows, f.cols, f.nb,
                                                           f.rec_pitch, f.e_pitch, W, ldw, vec);
  } else {
    int rc = allow_max_smem((const void*)decompress_kernel<12>, dev);
    if (rc) return rc;
    decompress_kernel<12><<<grid, kThreads, smem, stream>>>(rec, eplane, f.rows, f.cols, f.nb,
                                                            f.rec_pitch, f.e_pitch, W, ldw, vec);
  }
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace seedlm
