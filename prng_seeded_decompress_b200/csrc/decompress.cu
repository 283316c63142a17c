// decompress.cu -- W = the rebuilt weights, written out in fp32.
//
// Eq (1) of the paperhub.cn review thread, W_blk = U t, applied to every
// block.  A thread takes 4 consecutive blocks of a row (one 16-byte record
// load), rebuilds their weights exactly (see seedlm_device.cuh) and stores
// them with 16-byte streaming stores when the destination allows.  The kernel
// is bound by the 4 bytes per weight it writes, eight times the 0.5 bytes per
// weight it reads.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

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
                                            const uint8_t* __restrict__ eplane, int rec_pitch,
                                            int e_pitch, int r, int k) {
  Chunk ch;
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

// One thread per chunk of 4 blocks (grid-stride, next chunk loaded before
// the current one is rebuilt).  Chunks never straddle rows; blocks of a
// chunk at or past nb are skipped (rec_pitch covers the 16-byte load).
template <int C>
__global__ void __launch_bounds__(kThreads)
decompress_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane, int rows,
                  int cols, int nb, int rec_pitch, int e_pitch, float* __restrict__ W, int64_t ldw,
                  int vec) {
  // Jump tables: 32-bit words for C = 8 (stream bits 16..47 suffice), 64-bit
  // for C = 12 (bits 16..79).
  __shared__ __align__(16) unsigned char tab[512 * 8];
  uint32_t* t32 = reinterpret_cast<uint32_t*>(tab);
  uint2* t64 = reinterpret_cast<uint2*>(tab);
  for (int i = threadIdx.x; i < 512; i += kThreads) {
    uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
    if constexpr (C == 8)
      t32[i] = (uint32_t)v;
    else
      t64[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
  }
  __syncthreads();
  const int cpr = (nb + kRecs - 1) / kRecs;  // chunks per row
  const int64_t total = (int64_t)rows * cpr;
  const int64_t step = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (i >= total) return;
  int r = (int)(i / cpr), k = (int)(i - (int64_t)r * cpr);
  Chunk cur = load_chunk<C>(rec, eplane, rec_pitch, e_pitch, r, k);
  while (true) {
    const int64_t inext = i + step;
    int rn = 0, kn = 0;
    Chunk nxt;
    if (inext < total) {
      rn = (int)(inext / cpr);
      kn = (int)(inext - (int64_t)rn * cpr);
      nxt = load_chunk<C>(rec, eplane, rec_pitch, e_pitch, rn, kn);
    }
    const uint32_t words[kRecs] = {cur.rec.x, cur.rec.y, cur.rec.z, cur.rec.w};
#pragma unroll
    for (int q = 0; q < kRecs; ++q) {
      const int b = kRecs * k + q;
      if (b < nb) {
        float w[C];
        rebuild_block<C>(words[q], (cur.e >> (4 * q)) & 15u, t32, t64, w);
        float* dst = W + (size_t)r * (size_t)ldw + (size_t)b * C;
        const int j0 = b * C;
        if (vec && j0 + C <= cols) {
#pragma unroll
          for (int v = 0; v < C / 4; ++v)
            __stcs(reinterpret_cast<float4*>(dst) + v,
                   make_float4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]));
        } else {
#pragma unroll
          for (int c = 0; c < C; ++c)
            if (j0 + c < cols) dst[c] = w[c];
        }
      }
    }
    if (inext >= total) return;
    i = inext;
    r = rn;
    k = kn;
    cur = nxt;
  }
}

}  // namespace

int launch_decompress(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane, float* W,
                      int64_t ldw, cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t total = (int64_t)f.rows * ((f.nb + kRecs - 1) / kRecs);
  if (total == 0) return SEEDLM_OK;
  const int vec = ((reinterpret_cast<uintptr_t>(W) & 15u) == 0 && (ldw % 4) == 0) ? 1 : 0;
  int64_t want = (total + kThreads - 1) / kThreads;
  int64_t cap = (int64_t)dev.num_sms * 16;
  int grid = (int)(want < cap ? want : cap);
  if (f.C == 8)
    decompress_kernel<8><<<grid, kThreads, 0, stream>>>(rec, eplane, f.rows, f.cols, f.nb,
                                                        f.rec_pitch, f.e_pitch, W, ldw, vec);
  else
    decompress_kernel<12><<<grid, kThreads, 0, stream>>>(rec, eplane, f.rows, f.cols, f.nb,
                                                         f.rec_pitch, f.e_pitch, W, ldw, vec);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace seedlm
