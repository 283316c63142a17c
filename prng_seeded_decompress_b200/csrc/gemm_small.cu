// gemm_small.cu -- Y = X W^T for a small batch (1 <= M <= 64), CUDA cores.
//
// The same on-the-fly reconstruction as the GEMV, amortised over the M rows
// of X (paperhub.cn review thread: the rebuilt weights are used to compute the
// activations).  A CTA owns 32 rows of W and walks the columns in chunks of
// 192 (a multiple of both block lengths): it rebuilds the 32 x 192 tile into
// shared memory (exact fp32), stages the matching M x 192 slice of X as fp32,
// and every thread accumulates up to 8 outputs Y[m][r] in registers across
// all chunks.  Each rebuilt weight is therefore used M times.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

namespace {

constexpr int kThreads = 256;
constexpr int kTileRows = 32;
constexpr int kChunk = 192;
constexpr int kLd = kChunk + 1;  // padded row: lanes read distinct banks
constexpr int kMaxM = 64;

template <int C>
__global__ void __launch_bounds__(kThreads)
gemm_small_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane, int rows,
                  int cols, int nb, int rec_pitch, int e_pitch, const uint16_t* __restrict__ X,
                  int is_bf16, int M, float* __restrict__ Y) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* t32 = reinterpret_cast<uint32_t*>(smem);
  uint2* t64 = reinterpret_cast<uint2*>(smem);
  float* Wt = reinterpret_cast<float*>(smem + 512 * 8);
  float* Xt = Wt + kTileRows * kLd;
  for (int i = threadIdx.x; i < 512; i += kThreads) {
    uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
    if constexpr (C == 8)
      t32[i] = (uint32_t)v;
    else
      t64[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
  }
  const int row0 = blockIdx.x * kTileRows;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[kMaxM / 8];
#pragma unroll
  for (int k = 0; k < kMaxM / 8; ++k) acc[k] = 0.f;
  constexpr int kBlocks = kChunk / C;  // blocks per row per chunk
  for (int c0 = 0; c0 < cols; c0 += kChunk) {
    __syncthreads();  // previous chunk fully consumed (and tables written)
    for (int i = threadIdx.x; i < kTileRows * kBlocks; i += kThreads) {
      const int rr = i / kBlocks, bb = i - rr * kBlocks;
      const int r = row0 + rr, b = c0 / C + bb;
      float w[C];
      if (r < rows && b < nb) {
        const uint32_t word = __ldg(rec + (size_t)r * rec_pitch + b);
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
          const uint8_t eb = __ldg(eplane + (size_t)r * e_pitch + (b >> 1));
          const uint32_t e4 = (b & 1) ? (uint32_t)(eb >> 4) : (uint32_t)(eb & 15);
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
      } else {
#pragma unroll
        for (int c = 0; c < C; ++c) w[c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < C; ++c) Wt[rr * kLd + bb * C + c] = w[c];
    }
    for (int i = threadIdx.x; i < kMaxM * kChunk; i += kThreads) {
      const int m = i / kChunk, k = i - m * kChunk;
      const int j = c0 + k;
      Xt[m * kLd + k] = (m < M && j < cols) ? act_to_float(X[(size_t)m * cols + j], is_bf16) : 0.f;
    }
    __syncthreads();
    // Thread (warp, lane) owns row `lane` and batch rows warp, warp+8, ...
#pragma unroll
    for (int q = 0; q < kMaxM / 8; ++q) {
      const int m = warp + 8 * q;
      if (m < M) {
        float s = acc[q];
        const float* wr = Wt + lane * kLd;
        const float* xr = Xt + m * kLd;
#pragma unroll 8
        for (int k = 0; k < kChunk; ++k) s = fmaf(wr[k], xr[k], s);
        acc[q] = s;
      }
    }
  }
  const int r = row0 + lane;
  if (r < rows) {
#pragma unroll
    for (int q = 0; q < kMaxM / 8; ++q) {
      const int m = warp + 8 * q;
      if (m < M) Y[(size_t)m * rows + r] = acc[q];
    }
  }
}

}  // namespace

int launch_gemm_small(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                      const uint16_t* X, int is_bf16, int M, float* Y, cudaStream_t stream,
                      const DeviceInfo& dev) {
  if (f.rows == 0) return SEEDLM_OK;
  const size_t smem = 512 * 8 + (size_t)(kTileRows + kMaxM) * kLd * sizeof(float);
  const int grid = (f.rows + kTileRows - 1) / kTileRows;
  if (f.C == 8) {
    int rc_attr = allow_max_smem((const void*)gemm_small_kernel<8>, dev);
    if (rc_attr) return rc_attr;
    gemm_small_kernel<8><<<grid, kThreads, smem, stream>>>(rec, eplane, f.rows, f.cols, f.nb,
                                                          f.rec_pitch, f.e_pitch, X, is_bf16, M, Y);
  } else {
    int rc_attr = allow_max_smem((const void*)gemm_small_kernel<12>, dev);
    if (rc_attr) return rc_attr;
    gemm_small_kernel<12><<<grid, kThreads, smem, stream>>>(rec, eplane, f.rows, f.cols, f.nb,
                                                           f.rec_pitch, f.e_pitch, X, is_bf16, M,
                                                           Y);
  }
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace seedlm
