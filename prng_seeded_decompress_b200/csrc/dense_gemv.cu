// dense_gemv.cu -- y = W x with W stored dense in fp16: the memory-bound
// reference point the compressed GEMV is compared against (the pages compare
// SeedLM with an FP16 reference design; atlas.scime.ai, "Key results").
//
// One CTA of 16 warps per SM, persistent.  x is converted to fp32 into shared
// memory once per CTA.  A warp owns two rows at a time (row pairs are dealt
// out over all warps of the grid); each lane streams 16-byte chunks of both
// rows, four chunks per row in flight, and the row sums are reduced with warp
// shuffles.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

SEEDLM_CHECK_FLAG(dense)

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kUnroll = 4;

__device__ __forceinline__ float dot8(uint4 w, const float* xv) {
  const __half2* h = reinterpret_cast<const __half2*>(&w);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    s = fmaf(f.x, xv[2 * i], s);
    s = fmaf(f.y, xv[2 * i + 1], s);
  }
  return s;
}

__global__ void __launch_bounds__(kThreads, 1)
dense_gemv_f16_kernel(int rows, int cols, const uint16_t* __restrict__ W, int64_t ldw,
                      const uint16_t* __restrict__ x, float* __restrict__ y) {
  extern __shared__ __align__(16) float xs[];
  const int cols8 = (cols + 7) / 8 * 8;
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = seedlm_dynamic_smem_bytes() / 4;)
  for (int j = threadIdx.x; j < cols8; j += kThreads)
    if (SEEDLM_IN_BOUNDS(g_check_flag, j, xs_floats))
      xs[j] = j < cols ? __half2float(__ushort_as_half(x[j])) : 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarps;
  const int full8 = cols / 8;  // whole 16-byte chunks per row
  for (int r0 = 2 * gwarp; r0 < rows; r0 += 2 * nwarps) {
    const bool two = r0 + 1 < rows;
    const uint16_t* w0 = W + (size_t)r0 * (size_t)ldw;
    const uint16_t* w1 = two ? w0 + ldw : w0;
    float s0 = 0.f, s1 = 0.f;
    int k = lane;
    for (; k + 32 * (kUnroll - 1) < full8; k += 32 * kUnroll) {
      uint4 a[kUnroll], b[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        // The chunk's last element lies inside the row.
        const bool ok = SEEDLM_IN_BOUNDS(g_check_flag, 8 * (k + 32 * u) + 7, cols);
        a[u] = ok ? ld_stream_u4(w0 + 8 * (k + 32 * u)) : make_uint4(0u, 0u, 0u, 0u);
        b[u] = ok ? ld_stream_u4(w1 + 8 * (k + 32 * u)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const float* xv = xs + 8 * (k + 32 * u);
        s0 += dot8(a[u], xv);
        s1 += dot8(b[u], xv);
      }
    }
    for (; k < full8; k += 32) {
      if (!SEEDLM_IN_BOUNDS(g_check_flag, 8 * k + 7, cols)) continue;
      uint4 a = ld_stream_u4(w0 + 8 * k), b = ld_stream_u4(w1 + 8 * k);
      s0 += dot8(a, xs + 8 * k);
      s1 += dot8(b, xs + 8 * k);
    }
    for (int j = full8 * 8 + lane; j < cols; j += 32) {
      s0 = fmaf(__half2float(__ushort_as_half(w0[j])), xs[j], s0);
      s1 = fmaf(__half2float(__ushort_as_half(w1[j])), xs[j], s1);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (lane == 0) {
      if (SEEDLM_IN_BOUNDS(g_check_flag, r0, rows)) y[r0] = s0;
      if (two && SEEDLM_IN_BOUNDS(g_check_flag, r0 + 1, rows)) y[r0 + 1] = s1;
    }
  }
}

}  // namespace

int launch_dense_gemv_f16(int rows, int cols, const uint16_t* W, int64_t ldw, const uint16_t* x,
                          float* y, cudaStream_t stream, const DeviceInfo& dev) {
  if (rows == 0) return SEEDLM_OK;
  const size_t smem = (size_t)((cols + 7) / 8 * 8) * sizeof(float);
  if (smem > (size_t)dev.max_smem_optin) return SEEDLM_EUNSUPPORTED;
  int rc_attr = allow_max_smem((const void*)dense_gemv_f16_kernel, dev);
  if (rc_attr) return rc_attr;
  int pairs = (rows + 1) / 2;
  int want = (pairs + kWarps - 1) / kWarps;
  int grid = want < dev.num_sms ? want : dev.num_sms;
  dense_gemv_f16_kernel<<<grid, kThreads, smem, stream>>>(rows, cols, W, ldw, x, y);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace seedlm
