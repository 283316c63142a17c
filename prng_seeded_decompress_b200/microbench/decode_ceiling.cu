// decode_ceiling.cu -- the GEMV's per-block work with no memory traffic:
// records come from an LCG in registers, the decode reads lane-replicated
// tables at the GEMV's fixed shared addresses, and the rebuilt weights meet
// x values held in registers.  The rate (4-bit blocks per clock per SM) is
// the ceiling of the CUDA-core formulation; variants: 2 or 4 rows per step,
// packed vs scalar int->float adds, shifts as SHF or as the compiler's
// choice, and the core without the decode.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 \
//        -o decode_ceiling decode_ceiling.cu && ./decode_ceiling
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "../csrc/seedlm_device.cuh"

using namespace seedlm;

constexpr uint32_t kSmemBase = 1024, kTabJump = 0x10000, kTabCoef = 0x20000;

template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v; asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF)); return v;
}
template <uint32_t OFF>
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v; asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF)); return v;
}
__device__ __forceinline__ uint32_t shl_shf(uint32_t x, uint32_t n) {
  uint32_t d; asm("shf.l.clamp.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(0u), "r"(x), "r"(n)); return d;
}

template <int SHFMODE>
__device__ __forceinline__ BlockC8 dec(uint32_t rec, uint32_t lane4, uint32_t lane8) {
  BlockC8 b;
  b.lo = rec;
  b.hi = lds32<kTabJump>(prmt<0x5524u>(rec, lane4)) ^ lds32<kTabJump + 128>(prmt<0x5534u>(rec, lane4));
  uint32_t r4, r11;
  if (SHFMODE) { r4 = shl_shf(rec, 4); r11 = shl_shf(rec, 11); } else { r4 = rec << 4; r11 = rec << 11; }
  const uint2 c1 = lds64<kTabCoef>(prmt<0x5504u>(rec, lane8));
  const uint2 c2 = lds64<kTabCoef + 128>(prmt<0x5514u>(r4, lane8));
  b.a01 = c1.x; b.a23 = c2.x;
  const uint32_t e23 = r11 & 0x07800000u;
  b.init = (int32_t)(c1.y + c2.y - e23);
  b.negm = kNegMagicBits - e23;
  return b;
}

// ROWS rows x 2 blocks per lane per item, FP mode 0/1, SHF mode.
template <int ROWS, int FP, int SHFMODE, int NODEC>
__global__ void __launch_bounds__(768, 1) mb(int iters, unsigned long long* cyc, float* sink) {
  extern __shared__ __align__(16) unsigned char smem[];
  if ((uint32_t)__cvta_generic_to_shared(smem) != kSmemBase) { if (threadIdx.x == 0) cyc[blockIdx.x] = 1; return; }
  // fill tables with junk values (the values do not matter for timing)
  uint4* t = reinterpret_cast<uint4*>(smem + (kTabJump - kSmemBase));
  for (int i = threadIdx.x; i < 8192; i += blockDim.x) t[i] = make_uint4(i * 2654435761u, i, i ^ 0x5555u, i * 7u);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t lane4 = lane << 2, lane8 = (lane & 15) << 3;
  uint32_t st = threadIdx.x * 2654435761u + blockIdx.x;
  float2 xp[8];
  for (int c = 0; c < 8; ++c) xp[c] = make_float2(1e-3f * (c + 1), 2e-3f * (c + lane));
  float2 acc[ROWS];
  for (int j = 0; j < ROWS; ++j) acc[j] = make_float2(0.f, 0.f);
  const unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int j = 0; j < ROWS; ++j) {
      st = st * 1664525u + 1013904223u;
      const uint32_t ra = st, rb = st ^ 0x9e3779b9u;
      BlockC8 A, B;
      if (NODEC) {
        A.lo = ra; A.hi = rb; A.a01 = ra >> 3; A.a23 = rb >> 5; A.init = (int)(ra & 0xfff); A.negm = kNegMagicBits;
        B = A; B.lo = rb;
      } else {
        A = dec<SHFMODE>(ra, lane4, lane8);
        B = dec<SHFMODE>(rb, lane4, lane8);
      }
      const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
      float2 a = acc[j];
#define STEP(c) { const int32_t ba = weight_bits_c8<c>(A), bb = weight_bits_c8<c>(B); \
      if (FP == 1) { float2 w = make_float2(__int_as_float(ba) + negm.x, __int_as_float(bb) + negm.y); a = __ffma2_rn(w, xp[c], a); } \
      else { float2 w = make_float2(__int_as_float(ba), __int_as_float(bb)); a = __ffma2_rn(__fadd2_rn(w, negm), xp[c], a); } }
      STEP(0) STEP(1) STEP(2) STEP(3) STEP(4) STEP(5) STEP(6) STEP(7)
#undef STEP
      acc[j] = a;
    }
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  float s = 0.f;
  for (int j = 0; j < ROWS; ++j) s += acc[j].x + acc[j].y;
  if (s == 1.2345f) sink[threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
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
  const double blocks = (double)warps * 32 * iters * rows * 2;
  printf("%-36s warps %2d  blocks/clk/SM %.3f\n", name, warps, blocks / mx);
  cudaFree(cyc); cudaFree(sink);
}

int main() {
  // check the dynamic smem base first
  for (int w : {16, 24}) {
    run("4 rows fp0 shl", mb<4, 0, 0, 0>, 4, w);
    run("4 rows fp1 shl", mb<4, 1, 0, 0>, 4, w);
    run("4 rows fp0 shf", mb<4, 0, 1, 0>, 4, w);
    run("4 rows fp1 shf", mb<4, 1, 1, 0>, 4, w);
    run("2 rows fp0 shf", mb<2, 0, 1, 0>, 2, w);
    run("4 rows fp0 no decode (core only)", mb<4, 0, 0, 1>, 4, w);
    run("4 rows fp1 no decode (core only)", mb<4, 1, 0, 1>, 4, w);
  }
  return 0;
}
