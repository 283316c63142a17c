// amortised_ceiling.cu -- the 4-bit GEMV's per-block work in the
// "amortised" formulation, with no memory traffic, against the library's
// formulation measured the same way (decode_ceiling.cu).
//
// The amortised formulation moves the x-dependent part of the block dot to
// per-column-block tables shared by every row.  With b the block's stream
// bits and X~_m = sum_c x_c 2^(m-c) (0 <= m - c <= 15),
//   sum_c x_c state_{8p+c} = sum_m b_{8p+m} X~_m = T0[B_p] + T1[B_{p+1}] + T2[B_{p+2}],
// where B_k is stream byte k and T_j[v] = sum_k bit_k(v) X~_{8j+k} (three
// 256-entry tables per column block, built once from x).  Per (row, block)
// that leaves 9 table lookups, 6 adds, the coefficients as floats and
// y += 2^-e/32768 (q0 S0 + q1 S1 + q2 S2 - 32768 (q0+q1+q2) sum_c x_c).
//
// Layout here: lane l of a warp takes column block l, so the tables sit in
// lane-replicated 256-byte rows (T0, T1 at 0x10000, T2 at 0x20000) and each
// lookup is one conflict-free wavefront; the 64 KB of stream jump tables do
// not fit beside them, so stream bits 16..42 come from three passes of the
// register recurrence.  Records come from an LCG in registers.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//        -o amortised_ceiling amortised_ceiling.cu && ./amortised_ceiling
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "../csrc/seedlm_device.cuh"

using namespace seedlm;

constexpr uint32_t kSmemBase = 1024, kT01 = 0x10000, kT2 = 0x20000;

template <uint32_t OFF>
__device__ __forceinline__ float ldsf(uint32_t a) {
  float v; asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF)); return v;
}

// One pass of b[m+16] = b[m]^b[m+2]^b[m+3]^b[m+5] over a 32-bit word.
__device__ __forceinline__ uint32_t lfsr_pass(uint32_t x) {
  const uint32_t u = x ^ (x >> 2);
  return u ^ (u >> 3);
}

// float(q) for the signed byte k of s (sign-extended by prmt).
template <int K>
__device__ __forceinline__ float qf(uint32_t s) {
  constexpr uint32_t sel = ((8u | K) << 12) | ((8u | K) << 8) | ((8u | K) << 4) | K;
  return __int2float_rn((int32_t)prmt<sel>(s, 0u));
}

template <int ROWS>
__global__ void __launch_bounds__(512, 1) amortised(int iters, unsigned long long* cyc, float* sink) {
  extern __shared__ __align__(16) unsigned char smem[];
  if ((uint32_t)__cvta_generic_to_shared(smem) != kSmemBase) { if (threadIdx.x == 0) cyc[blockIdx.x] = 1; return; }
  float* t = reinterpret_cast<float*>(smem + (kT01 - kSmemBase));
  for (int i = threadIdx.x; i < 0x20000 / 4; i += blockDim.x) t[i] = 1e-3f * (float)(i & 1023);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t lane4 = lane << 2;
  const float xs = 1e-2f * (lane + 1);  // the column block's sum of x
  uint32_t st = threadIdx.x * 2654435761u + blockIdx.x;
  float acc[ROWS];
  for (int j = 0; j < ROWS; ++j) acc[j] = 0.f;
  const unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < ROWS; ++j) {
      st = st * 1664525u + 1013904223u;
      const uint32_t rec = st;  // seed in bits [16,32)
      const uint32_t t1 = lfsr_pass(rec);
      const uint32_t t2 = lfsr_pass(prmt<0x7632u>(rec, t1));
      const uint32_t hi = lfsr_pass(prmt<0x5432u>(rec, t2));  // stream bits 16..42
      const uint32_t a0 = prmt<0x5524u>(rec, lane4), a1 = prmt<0x5534u>(rec, lane4);
      const uint32_t a2 = prmt<0x5504u>(hi, lane4), a3 = prmt<0x5514u>(hi, lane4);
      const uint32_t a4 = prmt<0x5524u>(hi, lane4);
      const float s0 = ldsf<kT01>(a0) + ldsf<kT01 + 128>(a1) + ldsf<kT2>(a2);
      const float s1 = ldsf<kT01>(a1) + ldsf<kT01 + 128>(a2) + ldsf<kT2>(a3);
      const float s2 = ldsf<kT01>(a2) + ldsf<kT01 + 128>(a3) + ldsf<kT2>(a4);
      const uint32_t v = prmt<0x5140u>(rec, rec >> 4) & 0x0f0f0f0fu;  // q0, q1, q2, e
      const uint32_t s = sext_nibble_bytes(v);
      const float q0 = qf<0>(s), q1 = qf<1>(s), q2 = qf<2>(s);
      const float scale = __uint_as_float(0x38000000u - ((rec << 11) & 0x07800000u));  // 2^-(15+e)
      float d = q0 * s0;
      d = fmaf(q1, s1, d);
      d = fmaf(q2, s2, d);
      d = fmaf(q0 + q1 + q2, -32768.f * xs, d);
      acc[j] = fmaf(scale, d, acc[j]);
    }
  }
  __syncthreads();
  const unsigned long long t1c = clock64();
  float sum = 0.f;
  for (int j = 0; j < ROWS; ++j) sum += acc[j];
  if (sum == 1.2345f) sink[threadIdx.x] = sum;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1c - t0;
}

template <typename K>
void run(const char* name, K kern, int rows, int warps) {
  int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  const size_t smem = 0x30000 - kSmemBase;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  unsigned long long* cyc; float* sink;
  cudaMalloc(&cyc, 8 * sms); cudaMalloc(&sink, 4 * 1024);
  const int iters = 400;
  kern<<<sms, warps * 32, smem>>>(iters, cyc, sink);
  cudaDeviceSynchronize();
  kern<<<sms, warps * 32, smem>>>(iters, cyc, sink);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) { printf("%s: %s\n", name, cudaGetErrorString(e)); return; }
  unsigned long long h[256]; cudaMemcpy(h, cyc, 8 * sms, cudaMemcpyDeviceToHost);
  unsigned long long mx = 0; for (int i = 0; i < sms; ++i) mx = h[i] > mx ? h[i] : mx;
  const double blocks = (double)warps * 32 * iters * rows;
  printf("%-36s warps %2d  blocks/clk/SM %.3f\n", name, warps, blocks / mx);
  cudaFree(cyc); cudaFree(sink);
}

int main() {
  for (int w : {8, 16}) {
    run("amortised, 4 rows per step", amortised<4>, 4, w);
    run("amortised, 8 rows per step", amortised<8>, 8, w);
  }
  return 0;
}
