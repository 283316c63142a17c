// decompress.cu -- W = the rebuilt weights, written out in fp32.
//
// Eq (1) of the paperhub.cn review thread, W_blk = U t, applied to every
// block.  One thread per block: it decodes the record, rebuilds the C weights
// exactly (see seedlm_device.cuh) and stores them with 16-byte stores when the
// destination allows.  The kernel is bound by the 4 bytes per weight it
// writes, eight times the 0.5 bytes per weight it reads.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

namespace {

constexpr int kThreads = 256;

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
  const int64_t total = (int64_t)rows * nb;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * kThreads) {
    const int r = (int)(i / nb);
    const int b = (int)(i - (int64_t)r * nb);
    const uint32_t word = __ldg(rec + (size_t)r * rec_pitch + b);
    float w[C];
    if constexpr (C == 8) {
      const BlockC8 blk = decode_c8(word, t32, t32 + 256);
      const float negm = __uint_as_float(blk.negm);
      w[0] = __int_as_float(weight_bits_c8<0>(blk)) + negm;
      w[1] = __int_as_float(weight_bits_c8<1>(blk)) + negm;
      w[2] = __int_as_float(weight_bits_c8<2>(blk)) + negm;
      w[3] = __int_as_float(weight_bits_c8<3>(blk)) + negm;
      w[4] = __int_as_float(weight_bits_c8<4>(blk)) + negm;
      w[5] = __int_as_float(weight_bits_c8<5>(blk)) + negm;
      w[6] = __int_as_float(weight_bits_c8<6>(blk)) + negm;
      w[7] = __int_as_float(weight_bits_c8<7>(blk)) + negm;
    } else {
      const uint8_t eb = __ldg(eplane + (size_t)r * e_pitch + (b >> 1));
      const uint32_t e4 = (b & 1) ? (uint32_t)(eb >> 4) : (uint32_t)(eb & 15);
      const BlockC12 blk = decode_c12(word, e4, t64, t64 + 256);
      const float negm = __uint_as_float(blk.negm);
      w[0] = __int_as_float(weight_bits_c12<0>(blk)) + negm;
      w[1] = __int_as_float(weight_bits_c12<1>(blk)) + negm;
      w[2] = __int_as_float(weight_bits_c12<2>(blk)) + negm;
      w[3] = __int_as_float(weight_bits_c12<3>(blk)) + negm;
      w[4] = __int_as_float(weight_bits_c12<4>(blk)) + negm;
      w[5] = __int_as_float(weight_bits_c12<5>(blk)) + negm;
      w[6] = __int_as_float(weight_bits_c12<6>(blk)) + negm;
      w[7] = __int_as_float(weight_bits_c12<7>(blk)) + negm;
      w[8] = __int_as_float(weight_bits_c12<8>(blk)) + negm;
      w[9] = __int_as_float(weight_bits_c12<9>(blk)) + negm;
      w[10] = __int_as_float(weight_bits_c12<10>(blk)) + negm;
      w[11] = __int_as_float(weight_bits_c12<11>(blk)) + negm;
    }
    float* dst = W + (size_t)r * (size_t)ldw + (size_t)b * C;
    const int j0 = b * C;
    if (vec && j0 + C <= cols) {
#pragma unroll
      for (int q = 0; q < C / 4; ++q)
        __stcs(reinterpret_cast<float4*>(dst) + q,
               make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
    } else {
#pragma unroll
      for (int c = 0; c < C; ++c)
        if (j0 + c < cols) dst[c] = w[c];
    }
  }
}

}  // namespace

int launch_decompress(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane, float* W,
                      int64_t ldw, cudaStream_t stream, const DeviceInfo& dev) {
  const int64_t total = (int64_t)f.rows * f.nb;
  if (total == 0) return SEEDLM_OK;
  const int vec = ((reinterpret_cast<uintptr_t>(W) & 15u) == 0 && (ldw % 4) == 0) ? 1 : 0;
  int64_t want = (total + kThreads - 1) / kThreads;
  int64_t cap = (int64_t)dev.num_sms * 8;
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
