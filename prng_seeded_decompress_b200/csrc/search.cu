// search.cu -- exhaustive seed / coefficient / exponent search for blocks of
// any block size C, latent dimension P and seed width K: the design-space
// variants the pages discuss (paperhub.cn review thread, authors' replies on
// compression time against seed bit-width, block size and latent dimension;
// atlas.scime.ai summary, "Limitations": the design choices were explored on
// Gaussian weights).  The (8,3,16) and (12,4,16) formats have the faster
// tensor-core encoder in encode.cu; this one serves every other shape, on a
// flat list of blocks (no record packing, since K + 4P + 4 may exceed 32).
//
// The register: K bits, shifting right, the new top bit the parity of the
// tapped bits, state_0 = seed.  For K = 16 the taps are the workload's
// (bits 0, 2, 3, 5); for other K the pages give no polynomial, and the
// library takes the smallest odd tap mask whose register visits all 2^K - 1
// nonzero states (found by stepping it, once per K).  U(s)[c][p] =
// (state_{pC+c} - 2^(K-1)) / 2^(K-1).
//
// The search is the encoder's reading: t* = G^-1 U^T w (G = U^T U), for
// e = 15..0: q = clamp(round-half-even(t* 2^e), -8, 7), error
// ||w||^2 - 2^(1-e) q.(U^T w) + 2^(-2e) q^T G q, the minimum over seeds and
// exponents winning, ties to the smallest seed, then the largest e.  A
// candidate whose expanded error is within a margin of the lane's best is
// re-scored directly, sum_c (w_c - (U q)_c 2^-e)^2 with U regenerated from
// the register, so exact fits score exactly 0 and ties follow the rule.
//
// Two kernels, fp64 throughout: seed_tables_kernel (one thread per seed: U,
// G, G^-1 by Gauss-Jordan, H = G^-1 U^T, stored seed-minor so that a warp's
// lanes read consecutive seeds), then search_kernel (one warp per block,
// lanes striding over the seeds, a lexicographic warp argmin at the end).
// Both are instantiated for C in {8, 12, 16} and P in {2, 3, 4}, so every
// per-seed array lives in registers.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "seedlm_internal.h"

namespace seedlm {

namespace {

constexpr int kMaxP = 4, kMinK = 8, kMaxK = 20;
constexpr double kRescoreMargin = 1e-9;  // relative to ||w||^2

__host__ __device__ inline uint32_t lfsr_step(uint32_t s, int K, uint32_t taps) {
#ifdef __CUDA_ARCH__
  const uint32_t par = (uint32_t)__popc(s & taps) & 1u;
#else
  const uint32_t par = (uint32_t)__builtin_popcount(s & taps) & 1u;
#endif
  return (s >> 1) | (par << (K - 1));
}

// U(s) into u[c * P + p].
template <int C, int P>
__device__ __forceinline__ void basis(uint32_t seed, int K, uint32_t taps, double (&u)[C * P]) {
  const double half = (double)(1u << (K - 1));
  uint32_t s = seed;
#pragma unroll
  for (int k = 0; k < C * P; ++k) {
    const int p = k / C, c = k - p * C;
    u[c * P + p] = ((double)s - half) / half;
    s = lfsr_step(s, K, taps);
  }
}

// Row j of the per-seed table (H: P*C entries, then G: P*P), seed s >= 1.
__device__ __forceinline__ size_t tab_index(int j, uint32_t s, uint32_t nseeds) {
  return (size_t)j * nseeds + (s - 1);
}

template <int C, int P>
__global__ void seed_tables_kernel(int K, uint32_t taps, uint32_t nseeds, double* __restrict__ tab) {
  const uint32_t s = blockIdx.x * blockDim.x + threadIdx.x + 1;
  if (s > nseeds) return;
  double u[C * P], g[P * P], gi[P * P], m[P * P];
  basis<C, P>(s, K, taps, u);
#pragma unroll
  for (int a = 0; a < P; ++a)
#pragma unroll
    for (int b = 0; b < P; ++b) {
      double acc = 0.0;
#pragma unroll
      for (int c = 0; c < C; ++c) acc += u[c * P + a] * u[c * P + b];
      g[a * P + b] = acc;
      m[a * P + b] = acc;
      gi[a * P + b] = (a == b) ? 1.0 : 0.0;
    }
  // Gauss-Jordan (G is symmetric positive definite: U has full column rank
  // for every seed of the shapes instantiated here).
#pragma unroll
  for (int col = 0; col < P; ++col) {
    const double inv = 1.0 / m[col * P + col];
#pragma unroll
    for (int b = 0; b < P; ++b) {
      m[col * P + b] *= inv;
      gi[col * P + b] *= inv;
    }
#pragma unroll
    for (int a = 0; a < P; ++a) {
      if (a == col) continue;
      const double f = m[a * P + col];
#pragma unroll
      for (int b = 0; b < P; ++b) {
        m[a * P + b] -= f * m[col * P + b];
        gi[a * P + b] -= f * gi[col * P + b];
      }
    }
  }
  // H = G^-1 U^T (P x C), then G.
#pragma unroll
  for (int p = 0; p < P; ++p)
#pragma unroll
    for (int c = 0; c < C; ++c) {
      double acc = 0.0;
#pragma unroll
      for (int b = 0; b < P; ++b) acc += gi[p * P + b] * u[c * P + b];
      tab[tab_index(p * C + c, s, nseeds)] = acc;
    }
#pragma unroll
  for (int i = 0; i < P * P; ++i) tab[tab_index(P * C + i, s, nseeds)] = g[i];
}

struct Best {
  double err;
  uint32_t seed;
  int e;
  int q[kMaxP];
};

// (err, seed) lexicographically smaller; the exponent order is settled
// within a seed, where e runs downwards and only a strictly smaller error
// replaces the best.
__device__ __forceinline__ bool better(double err, uint32_t seed, const Best& b) {
  return err < b.err || (err == b.err && seed < b.seed);
}

template <int C, int P>
__global__ void search_kernel(int K, uint32_t taps, uint32_t nseeds, const double* __restrict__ tab,
                              const float* __restrict__ W, int64_t nblocks,
                              uint32_t* __restrict__ seed_out, int8_t* __restrict__ q_out,
                              uint8_t* __restrict__ e_out, double* __restrict__ err_out) {
  const int lane = threadIdx.x & 31;
  const int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (blk >= nblocks) return;  // warp-uniform
  double w[C];
  double ww = 0.0;
#pragma unroll
  for (int c = 0; c < C; ++c) {
    w[c] = (double)W[blk * C + c];
    ww += w[c] * w[c];
  }
  const double margin = kRescoreMargin * ww;
  Best best;
  best.err = INFINITY;
  best.seed = 0xffffffffu;
  best.e = 0;
#pragma unroll
  for (int p = 0; p < kMaxP; ++p) best.q[p] = 0;
  for (uint32_t s = lane + 1; s <= nseeds; s += 32) {
    double t[P], uw[P], g[P * P];
#pragma unroll
    for (int p = 0; p < P; ++p) {
      double acc = 0.0;
#pragma unroll
      for (int c = 0; c < C; ++c) acc += tab[tab_index(p * C + c, s, nseeds)] * w[c];
      t[p] = acc;
    }
#pragma unroll
    for (int i = 0; i < P * P; ++i) g[i] = tab[tab_index(P * C + i, s, nseeds)];
#pragma unroll
    for (int a = 0; a < P; ++a) {  // U^T w = G t*
      double acc = 0.0;
#pragma unroll
      for (int b = 0; b < P; ++b) acc += g[a * P + b] * t[b];
      uw[a] = acc;
    }
    for (int e = 15; e >= 0; --e) {
      const double sc = ldexp(1.0, e), isc = ldexp(1.0, -e);
      int q[P];
      bool zero = true;
#pragma unroll
      for (int p = 0; p < P; ++p) {
        const double v = fmin(fmax(rint(t[p] * sc), -8.0), 7.0);
        q[p] = (int)v;
        zero = zero && q[p] == 0;
      }
      double qu = 0.0, qgq = 0.0;
#pragma unroll
      for (int a = 0; a < P; ++a) {
        qu += q[a] * uw[a];
        double acc = 0.0;
#pragma unroll
        for (int b = 0; b < P; ++b) acc += g[a * P + b] * q[b];
        qgq += q[a] * acc;
      }
      double err = ww - 2.0 * isc * qu + isc * isc * qgq;
      if (err <= best.err + margin) {
        // Near or below the best: score it directly, U from the register.
        double rec[C];
#pragma unroll
        for (int c = 0; c < C; ++c) rec[c] = 0.0;
        const double half = (double)(1u << (K - 1));
        uint32_t st = s;
#pragma unroll
        for (int k = 0; k < C * P; ++k) {
          const int p = k / C, c = k - p * C;
          rec[c] += ((double)st - half) / half * q[p];
          st = lfsr_step(st, K, taps);
        }
        double d = 0.0;
#pragma unroll
        for (int c = 0; c < C; ++c) {
          const double r = w[c] - rec[c] * isc;
          d += r * r;
        }
        err = d;
        if (better(err, s, best)) {
          best.err = err;
          best.seed = s;
          best.e = e;
#pragma unroll
          for (int p = 0; p < P; ++p) best.q[p] = q[p];
        }
      }
      // Every q rounds to zero: all smaller exponents give this candidate.
      if (zero) break;
    }
  }
  // Warp argmin: smallest error, then smallest seed.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Best other;
    other.err = __shfl_xor_sync(0xffffffffu, best.err, o);
    other.seed = __shfl_xor_sync(0xffffffffu, best.seed, o);
    other.e = __shfl_xor_sync(0xffffffffu, best.e, o);
#pragma unroll
    for (int p = 0; p < kMaxP; ++p) other.q[p] = __shfl_xor_sync(0xffffffffu, best.q[p], o);
    if (better(other.err, other.seed, best)) best = other;
  }
  if (lane == 0) {
    seed_out[blk] = best.seed;
    e_out[blk] = (uint8_t)best.e;
#pragma unroll
    for (int p = 0; p < P; ++p) q_out[blk * P + p] = (int8_t)best.q[p];
    if (err_out) err_out[blk] = best.err;
  }
}

template <int C, int P>
int run_search(int K, uint32_t taps, const float* W, int64_t nblocks, uint32_t* seed, int8_t* q,
               uint8_t* e, double* err, cudaStream_t stream) {
  const uint32_t nseeds = (1u << K) - 1u;
  double* tab = nullptr;
  const size_t bytes = (size_t)(P * C + P * P) * nseeds * sizeof(double);
  int rc = record_cuda_error(cudaMallocAsync(reinterpret_cast<void**>(&tab), bytes, stream));
  if (rc) return rc;
  seed_tables_kernel<C, P><<<(nseeds + 127) / 128, 128, 0, stream>>>(K, taps, nseeds, tab);
  count_launch();
  rc = record_cuda_error(cudaGetLastError());
  if (!rc) {
    const int warps = 4;
    const int64_t grid = (nblocks + warps - 1) / warps;
    search_kernel<C, P><<<(unsigned)grid, warps * 32, 0, stream>>>(K, taps, nseeds, tab, W,
                                                                   nblocks, seed, q, e, err);
    count_launch();
    rc = record_cuda_error(cudaGetLastError());
  }
  const int rc_free = record_cuda_error(cudaFreeAsync(tab, stream));
  return rc ? rc : rc_free;
}

template <int C>
int dispatch_p(int P, int K, uint32_t taps, const float* W, int64_t n, uint32_t* seed, int8_t* q,
               uint8_t* e, double* err, cudaStream_t st) {
  switch (P) {
    case 2: return run_search<C, 2>(K, taps, W, n, seed, q, e, err, st);
    case 3: return run_search<C, 3>(K, taps, W, n, seed, q, e, err, st);
    case 4: return run_search<C, 4>(K, taps, W, n, seed, q, e, err, st);
    default: return SEEDLM_EUNSUPPORTED;
  }
}

}  // namespace

// Taps of the K-bit register (0 if K is outside [kMinK, kMaxK]).
uint32_t lfsr_taps(int K) {
  if (K < kMinK || K > kMaxK) return 0;
  if (K == 16) return 0x2Du;
  static std::mutex m;
  static uint32_t cache[kMaxK + 1] = {};
  std::lock_guard<std::mutex> lock(m);
  if (!cache[K]) {
    const uint32_t full = (1u << K) - 1u;
    for (uint32_t taps = 1; taps < (1u << K) && !cache[K]; taps += 2) {
      uint32_t s = 1, n = 0;
      do {
        s = lfsr_step(s, K, taps);
        ++n;
      } while (s != 1u && n <= full);
      if (n == full) cache[K] = taps;
    }
  }
  return cache[K];
}

int launch_search(int C, int P, int K, const float* W, int64_t nblocks, uint32_t* seed,
                  int8_t* q, uint8_t* e, double* err, cudaStream_t stream) {
  const uint32_t taps = lfsr_taps(K);
  if (!taps) return SEEDLM_EUNSUPPORTED;
  switch (C) {
    case 8: return dispatch_p<8>(P, K, taps, W, nblocks, seed, q, e, err, stream);
    case 12: return dispatch_p<12>(P, K, taps, W, nblocks, seed, q, e, err, stream);
    case 16: return dispatch_p<16>(P, K, taps, W, nblocks, seed, q, e, err, stream);
    default: return SEEDLM_EUNSUPPORTED;
  }
}

bool search_shape_ok(int C, int P, int K) {
  return (C == 8 || C == 12 || C == 16) && P >= 2 && P <= 4 && K >= kMinK && K <= kMaxK;
}

}  // namespace seedlm

using namespace seedlm;

extern "C" {

SEEDLM_API int seedlm_search_blocks(int32_t C, int32_t P, int32_t K, const float* W,
                                    int64_t nblocks, uint32_t* seed, int8_t* q, uint8_t* e,
                                    double* err, seedlm_stream stream) {
  if (!search_shape_ok(C, P, K)) return SEEDLM_EUNSUPPORTED;
  if (nblocks < 0 || nblocks > (int64_t)0x7fffffff * 4) return SEEDLM_EINVAL;
  if (nblocks == 0) return SEEDLM_OK;
  if (!W || !aligned(W, 4) || !seed || !aligned(seed, 4) || !q || !e) return SEEDLM_EINVAL;
  if (err && !aligned(err, 8)) return SEEDLM_EINVAL;
  DeviceInfo dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  return launch_search(C, P, K, W, nblocks, seed, q, e, err, (cudaStream_t)stream);
}

SEEDLM_API uint32_t seedlm_lfsr_taps(int32_t K) { return lfsr_taps(K); }

}  // extern "C"
