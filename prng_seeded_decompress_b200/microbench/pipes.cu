// pipes.cu -- issue rates of the instructions the SeedLM rebuild uses, alone
// and mixed: warp-instructions per clock per SM for dp2a (IDP), funnel shift
// (SHF), LOP3, FFMA, packed FFMA2 / FADD2, and shared-memory loads from a
// 256-entry table at random indices against a lane-replicated copy.  Each
// thread runs 8 independent chains so that latency does not limit the rate;
// cycles come from clock64 over the timed loop, the maximum over CTAs.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -o pipes pipes.cu && ./pipes
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>

#define NCH 8
__device__ __forceinline__ int dp2a(uint32_t a, uint32_t b, int c) {
  int d; asm volatile("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c)); return d;
}
__device__ __forceinline__ uint32_t shf(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t d; asm volatile("shf.r.wrap.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(s)); return d;
}
__device__ __forceinline__ float ffma(float a, float b, float c) {
  float d; asm volatile("fma.rn.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c)); return d;
}
__device__ __forceinline__ float fadd(float a, float b) {
  float d; asm volatile("add.rn.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b)); return d;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d; asm volatile("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c)); return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d; asm volatile("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b)); return d;
}
__device__ __forceinline__ uint32_t lop3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d; asm volatile("lop3.b32 %0, %1, %2, %3, 0x96;" : "=r"(d) : "r"(a), "r"(b), "r"(c)); return d;
}
__device__ __forceinline__ uint32_t iadd3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d; asm volatile("add.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b)); asm volatile("add.u32 %0, %0, %1;" : "+r"(d) : "r"(c)); return d;
}

// Mix: counts per iteration per chain.
template <int nIDP, int nSHF, int nFFMA, int nFADD, int nFFMA2, int nFADD2, int nLOP3>
__global__ void mix_kernel(int iters, uint32_t seed, unsigned long long* cyc, uint32_t* sink) {
  uint32_t ia[NCH]; float fa[NCH]; uint64_t pa[NCH]; uint32_t la[NCH];
  for (int k = 0; k < NCH; ++k) { ia[k] = seed * (k + 1) + threadIdx.x; fa[k] = (float)(k + threadIdx.x) * 1e-3f; pa[k] = ((uint64_t)__float_as_uint(fa[k]) << 32) | __float_as_uint(fa[k]); la[k] = ia[k] ^ 0x5555; }
  const uint32_t b = seed | 0x01010101u;
  const float fx = 0.999f; const uint64_t px = ((uint64_t)__float_as_uint(fx) << 32) | __float_as_uint(fx);
  __syncthreads();
  unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
#pragma unroll
      for (int j = 0; j < nIDP; ++j) ia[k] = dp2a(ia[k], b, (int)ia[k]);
#pragma unroll
      for (int j = 0; j < nSHF; ++j) la[k] = shf(la[k], ia[k], 3);
#pragma unroll
      for (int j = 0; j < nLOP3; ++j) la[k] = lop3(la[k], b, ia[k]);
#pragma unroll
      for (int j = 0; j < nFFMA; ++j) fa[k] = ffma(fa[k], fx, 1e-7f);
#pragma unroll
      for (int j = 0; j < nFADD; ++j) fa[k] = fadd(fa[k], 1e-7f);
#pragma unroll
      for (int j = 0; j < nFFMA2; ++j) pa[k] = ffma2(pa[k], px, px);
#pragma unroll
      for (int j = 0; j < nFADD2; ++j) pa[k] = fadd2(pa[k], px);
    }
  }
  __syncthreads();
  unsigned long long t1 = clock64();
  uint32_t s = 0;
  for (int k = 0; k < NCH; ++k) s += ia[k] + la[k] + __float_as_uint(fa[k]) + (uint32_t)pa[k] + (uint32_t)(pa[k] >> 32);
  if (s == 0x12345678u) sink[threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

// Random LDS from a 256-entry table (conflicts) vs a lane-replicated one.
template <int REPL>
__global__ void lds_kernel(int iters, uint32_t seed, unsigned long long* cyc, uint32_t* sink) {
  __shared__ uint32_t tab[256 * 32];
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) tab[i] = i * 2654435761u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  uint32_t x[NCH];
  for (int k = 0; k < NCH; ++k) x[k] = (seed + threadIdx.x * 7919u + k * 104729u) * 2654435761u;
  unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      uint32_t idx = (x[k] >> 13) & 255u;   // random-looking index, in [0,256)
      uint32_t v = REPL ? tab[idx * 32 + lane] : tab[idx];
      x[k] = x[k] * 1664525u + v;          // next index depends on the load
    }
  }
  __syncthreads();
  unsigned long long t1 = clock64();
  uint32_t s = 0;
  for (int k = 0; k < NCH; ++k) s += x[k];
  if (s == 0x12345678u) sink[threadIdx.x] = s;
  if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}

template <typename K>
void run(const char* name, K kern, int instr_per_chain_iter, int threads) {
  int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  unsigned long long* cyc; uint32_t* sink;
  cudaMalloc(&cyc, sizeof(unsigned long long) * sms); cudaMalloc(&sink, 4 * 1024);
  const int iters = 2000;
  kern<<<sms, threads>>>(iters, 12345u, cyc, sink);
  cudaDeviceSynchronize();
  kern<<<sms, threads>>>(iters, 12345u, cyc, sink);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) { printf("%s: error %s\n", name, cudaGetErrorString(e)); return; }
  unsigned long long h[1024]; cudaMemcpy(h, cyc, sizeof(unsigned long long) * sms, cudaMemcpyDeviceToHost);
  unsigned long long mx = 0; for (int i = 0; i < sms; ++i) if (h[i] > mx) mx = h[i];
  double warp_instr = (double)(threads / 32) * iters * NCH * instr_per_chain_iter;
  printf("%-34s warps/SM %2d  warp-instr/clk/SM %.3f\n", name, threads / 32, warp_instr / (double)mx);
  cudaFree(cyc); cudaFree(sink);
}

int main() {
  for (int threads : {512, 1024}) {
    run("IDP", mix_kernel<1, 0, 0, 0, 0, 0, 0>, 1, threads);
    run("SHF", mix_kernel<0, 1, 0, 0, 0, 0, 0>, 1, threads);
    run("LOP3", mix_kernel<0, 0, 0, 0, 0, 0, 1>, 1, threads);
    run("FFMA", mix_kernel<0, 0, 1, 0, 0, 0, 0>, 1, threads);
    run("FFMA2", mix_kernel<0, 0, 0, 0, 1, 0, 0>, 1, threads);
    run("IDP+FFMA", mix_kernel<1, 0, 1, 0, 0, 0, 0>, 2, threads);
    run("IDP+FFMA2", mix_kernel<1, 0, 0, 0, 1, 0, 0>, 2, threads);
    run("IDP+SHF", mix_kernel<1, 1, 0, 0, 0, 0, 0>, 2, threads);
    run("2IDP+SHF+FADD+FFMA", mix_kernel<2, 1, 1, 1, 0, 0, 0>, 5, threads);
    run("4IDP+2SHF+FADD2+FFMA2", mix_kernel<4, 2, 0, 0, 1, 1, 0>, 8, threads);
    run("4IDP+2SHF+2FADD+2FFMA", mix_kernel<4, 2, 2, 2, 0, 0, 0>, 10, threads);
    run("4IDP+2SHF+FADD2+2FFMA", mix_kernel<4, 2, 2, 0, 0, 1, 0>, 9, threads);
    run("4IDP+2SHF+2FADD+FFMA2", mix_kernel<4, 2, 0, 2, 1, 0, 0>, 9, threads);
    run("IDP+FFMA+SHF+LOP3", mix_kernel<1, 1, 1, 0, 0, 0, 1>, 4, threads);
    run("LDS random 256", lds_kernel<0>, 1, threads);
    run("LDS lane-replicated", lds_kernel<1>, 1, threads);
  }
  return 0;
}
