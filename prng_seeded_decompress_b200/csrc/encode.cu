// encode.cu -- the encoder side of the format: for every block of W, the
// seed, quantised coefficients and exponent that reconstruct it best.
//
// SeedLM (paperhub.cn review thread, authors' replies on the cost of
// parameter optimisation): each block is matched against every seed's
// pseudo-random matrix U(s) (C x P), the coefficients are fitted and
// quantised, and the seed with the smallest reconstruction error wins; the
// search is parallel over blocks and seeds, with per-seed data computed once
// and cached.  The pages fix no exponent or rounding rule; the reading used
// throughout this library:
//
//   t*(s) = pinv(U(s)) w              (U(s) has full column rank for every s,
//                                      so pinv(U) w = G^-1 U^T w, G = U^T U)
//   q(s, e) = clamp(round-half-even(t* 2^e), -8, 7),  e = 0..15
//   err(s, e) = ||w - U(s) q 2^-e||^2
//
// and the minimum over (s, e) wins, ties going to the smallest seed, then the
// largest exponent.  A tail block (cols not a multiple of C) is fitted with
// its missing weights taken as zero.
//
// Two kernels.  basis_table_kernel computes, once per call, an orthonormal
// basis Q(s) of every seed's column space (Gram-Schmidt in fp64, each column
// orthogonalised twice) and stores it rounded to fp32: one float4 per row c
// of U, (Q[c][0], Q[c][1], Q[c][2], Q[c][3]) for P = 4 and
// (Q[c][0], Q[c][1], Q[c][2], Q[c][2]) for P = 3.
//
// encode_kernel: one thread owns two neighbouring blocks of a row (for C = 12
// the two that share an exponent byte).  A CTA streams the table through
// shared memory in chunks of 128 seeds (cp.async, double-buffered), and for
// every seed each thread first evaluates, in fp32, the least-squares residual
//   r(s) = ||w||^2 - ||Q(s)^T w||^2,
// a lower bound on the error of every quantised candidate of that seed.  Only
// when r(s) is not above the block's best error so far plus a margin does the
// thread score the seed exactly (score_seed: fp64, U, G exact, G^-1 by
// Gauss-Jordan, the exponents in descending order with the expansion
//   err = ||w||^2 - 2^(1-e) q.(U^T w) + 2^(-2e) q^T G q ).
// On Gaussian blocks about 3 in 10^4 seeds get that far, so the search costs
// one fp32 projection per seed and block: 3 (C = 8) or 4 (C = 12) packed
// fp32x2 FMAs per basis row for both blocks, on a row read once.
//
// The filter never changes the result.  The block is scaled by 2^-E (exact)
// so that max|w| lies in [1, 2).  With u = 2^-24, each fp32 coordinate of
// Q^T w is within (C + 1) u ||w|| of the exact one (C fused products, plus
// the rounding of Q to fp32; the columns of Q have unit norm), so the squared
// norm is within about 2 sqrt(P) (C + 1) u ||w||^2 + P u ||w||^2, and ||w||^2
// in fp32 within C u ||w||^2: |r_fp32 - r| < 5e-6 ||w||^2 for both formats.
// The basis itself is orthonormal to fp64 rounding, and spans U(s)'s column
// space to within kappa(U) 2^-53 < 1e-10 (kappa(U) < 4e5 over all seeds), so
// a seed is skipped only if r_fp32 > best + 3e-5 ||w||^2, where no candidate
// of it can reach the best error (candidates are compared with strict <).
// The winner's error is recomputed directly at the end.
#include <cuda_runtime.h>

#include <cmath>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

SEEDLM_CHECK_FLAG(encode)

namespace {

constexpr int kEncThreads = 128;
constexpr int kNumSeeds = 65535;
constexpr int kTableRows = 65536;  // row i holds seed i + 1; the last row is zero padding
constexpr int kChunk = 128;        // seeds per shared-memory chunk
constexpr int kChunks = kTableRows / kChunk;
constexpr double kPruneMargin = 3e-5;  // relative to ||w||^2, six times the fp32 error bound
#ifndef SEEDLM_ENC_GROUP
#define SEEDLM_ENC_GROUP 4
#endif
constexpr int kGroup = SEEDLM_ENC_GROUP;  // seeds tested per survivor branch

// The seed's bit stream, bits [0, 64): state_k = bits [k, k + 16).
__device__ __forceinline__ uint64_t seed_stream(uint32_t seed) {
  const uint64_t ext = kStreamTables.lo[seed & 0xffu] ^ kStreamTables.hi[seed >> 8];
  return (uint64_t)seed | (ext << 16);
}

// U(seed)[c][p] = (state_{pC + c} - 32768) / 32768.
template <int C, int P>
__device__ __forceinline__ double basis_entry(uint64_t stream, int c, int p) {
  const int k = p * C + c;
  const int state = (int)((stream >> k) & 0xffffu);
  return (double)(state - 32768) * (1.0 / 32768.0);
}

// Inverse of a symmetric positive definite P x P matrix by Gauss-Jordan
// elimination (no pivoting needed for SPD).
template <int P>
__device__ void spd_inverse(const double* g, double* gi) {
  double a[P][2 * P];
#pragma unroll
  for (int i = 0; i < P; ++i)
#pragma unroll
    for (int j = 0; j < P; ++j) {
      a[i][j] = g[i * P + j];
      a[i][P + j] = (i == j) ? 1.0 : 0.0;
    }
#pragma unroll
  for (int k = 0; k < P; ++k) {
    const double inv = 1.0 / a[k][k];
#pragma unroll
    for (int j = 0; j < 2 * P; ++j) a[k][j] *= inv;
#pragma unroll
    for (int i = 0; i < P; ++i) {
      if (i == k) continue;
      const double f = a[i][k];
#pragma unroll
      for (int j = 0; j < 2 * P; ++j) a[i][j] -= f * a[k][j];
    }
  }
#pragma unroll
  for (int i = 0; i < P; ++i)
#pragma unroll
    for (int j = 0; j < P; ++j) gi[i * P + j] = a[i][P + j];
}

// fp64 data of one seed for exact scoring: G = U^T U (exact; row-major,
// upper triangle used) and G^-1 (Gauss-Jordan), padded to 20 or 32 doubles.
template <int P>
struct SeedExact {
  static constexpr int kDoubles = (2 * P * P + 3) / 4 * 4;
  static_assert(kDoubles >= 2 * P * P, "G and G^-1 fit one row");
};

// Row i of the tables: the orthonormal basis of seed i + 1, one float4 per
// row c of U (see the file comment), and its G and G^-1.
template <int C, int P>
__global__ void __launch_bounds__(256) basis_table_kernel(float4* __restrict__ table,
                                                          double* __restrict__ exact) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= kTableRows) return;
  float4* out = table + (size_t)i * C;
  if (i >= kNumSeeds) {
#pragma unroll
    for (int c = 0; c < C; ++c) out[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const uint64_t st = seed_stream((uint32_t)(i + 1));
  double q[C][P];
#pragma unroll
  for (int c = 0; c < C; ++c)
#pragma unroll
    for (int p = 0; p < P; ++p) q[c][p] = basis_entry<C, P>(st, c, p);
  {
    double g[P * P], gi[P * P];
#pragma unroll
    for (int p = 0; p < P; ++p)
#pragma unroll
      for (int r = 0; r < P; ++r) {
        double acc = 0.0;
#pragma unroll
        for (int c = 0; c < C; ++c) acc = fma(q[c][p], q[c][r], acc);  // exact
        g[p * P + r] = acc;
      }
    spd_inverse<P>(g, gi);
    double* ex = exact + (size_t)i * SeedExact<P>::kDoubles;
#pragma unroll
    for (int k = 0; k < P * P; ++k) {
      ex[k] = g[k];
      ex[P * P + k] = gi[k];
    }
  }
#pragma unroll
  for (int p = 0; p < P; ++p) {
#pragma unroll
    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
      for (int j = 0; j < p; ++j) {
        double d = 0.0;
#pragma unroll
        for (int c = 0; c < C; ++c) d = fma(q[c][j], q[c][p], d);
#pragma unroll
        for (int c = 0; c < C; ++c) q[c][p] = fma(-d, q[c][j], q[c][p]);
      }
    double n = 0.0;
#pragma unroll
    for (int c = 0; c < C; ++c) n = fma(q[c][p], q[c][p], n);
    const double inv = 1.0 / sqrt(n);
#pragma unroll
    for (int c = 0; c < C; ++c) q[c][p] *= inv;
  }
#pragma unroll
  for (int c = 0; c < C; ++c)
    out[c] = make_float4((float)q[c][0], (float)q[c][1], (float)q[c][2], (float)q[c][P - 1]);
}

// One block's search state, in shared memory where the whole warp can read
// it: the best candidate so far, and what exact scoring needs (||w||^2 in
// fp64, where the weights are, how many of them the row has).
template <int P>
struct BlockSlot {
  double err;
  double ww;
  const float* wsrc;
  uint32_t seed;
  int e;
  int q[P];
  int nvalid;
};

// The filter threshold of a block in its scaled domain (rounded up): a seed
// whose fp32 residual exceeds it cannot beat the best error.  Once the best
// error is 0 nothing can (strict <).
__device__ __forceinline__ float prune_threshold(double best, double ww, double s2) {
  if (best == 0.0) return -INFINITY;
  return __double2float_ru((best + kPruneMargin * ww) * s2);
}

// A seed's best candidate for one block, scored exactly in fp64: err and
// (e, q) packed as e | q_p << (4 + 4p) (q as 4-bit two's complement).
struct Cand {
  double err;
  uint32_t eq;
};

template <int C, int P>
__device__ __noinline__ Cand seed_candidate(uint32_t seed, const float* __restrict__ wsrc,
                                            int nvalid, double ww,
                                            const double* __restrict__ exact) {
  double w[C];
#pragma unroll
  for (int c = 0; c < C; ++c) w[c] = c < nvalid ? (double)wsrc[c] : 0.0;
  const uint64_t st = seed_stream(seed);
  const double* ex = exact + (size_t)(seed - 1) * SeedExact<P>::kDoubles;
  double g[P * P], gi[P * P], b[P], t[P];
#pragma unroll
  for (int k = 0; k < P * P; ++k) {
    g[k] = __ldg(ex + k);
    gi[k] = __ldg(ex + P * P + k);
  }
#pragma unroll
  for (int p = 0; p < P; ++p) {
    double acc = 0.0;
#pragma unroll
    for (int c = 0; c < C; ++c) acc = fma(basis_entry<C, P>(st, c, p), w[c], acc);
    b[p] = acc;
  }
#pragma unroll
  for (int p = 0; p < P; ++p) {
    double acc = 0.0;
#pragma unroll
    for (int r = 0; r < P; ++r) acc = fma(gi[p * P + r], b[r], acc);
    t[p] = acc;
  }
  Cand best{INFINITY, 15u};
  // Exponents in descending order: on an exact tie the larger e, met first,
  // stays.  |t* 2^e| shrinks with e, so once every q rounds to 0 all smaller
  // exponents give that same candidate (error ||w||^2): the loop ends there.
  for (int e = 15; e >= 0; --e) {
    const double sc = (double)(1 << e), inv = 1.0 / (double)(1 << e);
    double q[P];
    bool zero = true;
#pragma unroll
    for (int p = 0; p < P; ++p) {
      q[p] = fmin(fmax(rint(t[p] * sc), -8.0), 7.0);
      zero = zero && q[p] == 0.0;
    }
    // q.b and q^T G q (G symmetric: diagonal once, off-diagonal twice).
    double qb = 0.0, qgq = 0.0;
#pragma unroll
    for (int p = 0; p < P; ++p) {
      qb = fma(q[p], b[p], qb);
      double row = 0.5 * g[p * P + p] * q[p];
#pragma unroll
      for (int r = p + 1; r < P; ++r) row = fma(g[p * P + r], q[r], row);
      qgq = fma(q[p], row, qgq);
    }
    const double err = fma(2.0 * inv * inv, qgq, fma(-2.0 * inv, qb, ww));
    if (err < best.err) {
      best.err = err;
      uint32_t eq = (uint32_t)e;
#pragma unroll
      for (int p = 0; p < P; ++p) eq |= ((uint32_t)(int)q[p] & 15u) << (4 + 4 * p);
      best.eq = eq;
    }
    if (zero) break;
  }
  return best;
}

// Per-warp queue of (seed, block) pairs the filter let through, scored 32 at
// a time with every lane busy.  Entry: seed | lane << 16 | k << 21 (block k
// of that lane).
constexpr int kQueue = 96;  // < 32 left over + at most 64 added per seed
struct WarpQueue {
  uint32_t ent[kQueue];
  double err[32];
  uint32_t eq[32];
};

// Scores the queued pairs in batches of 32 (all of them if min_batch is 1,
// else while at least min_batch remain) and merges each result into its
// block's slot in queue order -- ascending seeds for every block, so a
// strictly smaller error replaces the best exactly as a sequential scan
// would.  Called by the whole warp; returns the entries left.
template <int C, int P>
__device__ __noinline__ int drain_queue(WarpQueue* wq, int count, int min_batch,
                                        BlockSlot<P>* wslots, const double* __restrict__ exact,
                                        int lane) {
  int base = 0;
  while (count - base > 0 && count - base >= min_batch) {
    const int n = min(32, count - base);
    if (lane < n) {
      const uint32_t en = wq->ent[base + lane];
      const BlockSlot<P>& bs = wslots[2 * ((en >> 16) & 31u) + (en >> 21)];
      const Cand cd = seed_candidate<C, P>(en & 0xffffu, bs.wsrc, bs.nvalid, bs.ww, exact);
      wq->err[lane] = cd.err;
      wq->eq[lane] = cd.eq;
    }
    __syncwarp();
    for (int i = 0; i < n; ++i) {
      const uint32_t en = wq->ent[base + i];
      if (((en >> 16) & 31u) == (uint32_t)lane) {
        BlockSlot<P>& bs = wslots[2 * lane + (en >> 21)];
        if (wq->err[i] < bs.err) {
          const uint32_t eq = wq->eq[i];
          bs.err = wq->err[i];
          bs.seed = en & 0xffffu;
          bs.e = (int)(eq & 15u);
#pragma unroll
          for (int p = 0; p < P; ++p) bs.q[p] = ((int)(eq << (24 - 4 * p))) >> 28;
        }
      }
    }
    __syncwarp();
    base += n;
  }
  const int left = count - base;
  if (base > 0) {
    const uint32_t v = lane < left ? wq->ent[base + lane] : 0u;
    __syncwarp();
    if (lane < left) wq->ent[lane] = v;
  }
  __syncwarp();
  return left;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Chunk k of the table (kChunk seeds x C float4, contiguous) into buf.
template <int C>
__device__ __forceinline__ void load_chunk(float4* buf, const float4* __restrict__ table, int k,
                                           int tid) {
  const float4* src = table + (size_t)k * kChunk * C;
#pragma unroll
  for (int i = 0; i < C; ++i) {
    const int j = tid + i * kEncThreads;  // kChunk * C = C * kEncThreads float4
    if (SEEDLM_IN_BOUNDS(g_check_flag, (size_t)k * kChunk * C + j, (size_t)kTableRows * C))
      cp_async16(buf + j, src + j);
  }
}

template <int C, int P>
__global__ void __launch_bounds__(kEncThreads)
encode_kernel(const float* __restrict__ W, int64_t ldw, int rows, int cols, int nb,
              int rec_pitch, int e_pitch, uint32_t* __restrict__ rec,
              uint8_t* __restrict__ eplane, double* __restrict__ err_out, long long n_items,
              const float4* __restrict__ table, const double* __restrict__ exact) {
  static_assert(kChunk == kEncThreads, "one float4 per thread and basis row");
  static_assert(kChunk % kGroup == 0, "whole seed groups per chunk");
  extern __shared__ __align__(16) unsigned char smem[];
  float4* qbuf = reinterpret_cast<float4*>(smem);  // [2][kChunk * C]
  BlockSlot<P>* slots =
      reinterpret_cast<BlockSlot<P>*>(smem + 2 * kChunk * C * sizeof(float4));  // [threads][2]
  WarpQueue* queues = reinterpret_cast<WarpQueue*>(slots + 2 * kEncThreads);  // [warps]
  const int tid = threadIdx.x, lane = tid & 31;
  WarpQueue* wq = queues + (tid >> 5);
  BlockSlot<P>* wslots = slots + 2 * (tid & ~31);  // this warp's 64 slots
  load_chunk<C>(qbuf, table, 0, tid);
  cp_async_commit();

  const int ipr = (nb + 1) / 2;  // items (block pairs) per row
  const long long item = (long long)blockIdx.x * kEncThreads + tid;
  const bool active = item < n_items;
  const int row = active ? (int)(item / ipr) : 0;
  const int b0 = active ? (int)(item - (long long)row * ipr) * 2 : 0;

  // Per block: the weights scaled by 2^-E (max |w| in [1, 2)) as (w, w)
  // pairs, ||w||^2 in fp64 and in the scaled fp32 domain, 2^-2E, the filter
  // threshold, and where the weights are in W.
  float2 wd[2][C];
  float ww32[2], thr[2];
  double ww64[2], s2[2];
  const float* wsrc[2];
  int nvalid[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int blk = b0 + k;
    const bool valid = active && blk < nb;
    nvalid[k] = valid ? min(C, cols - blk * C) : 0;
    wsrc[k] = W + (size_t)row * ldw + (size_t)blk * C;
    if (nvalid[k] > 0 &&
        !SEEDLM_IN_BOUNDS(g_check_flag, (size_t)row * ldw + (size_t)blk * C + nvalid[k] - 1,
                          (size_t)(rows - 1) * ldw + cols))
      nvalid[k] = 0;
    float w[C];
    float maxabs = 0.f;
    double acc = 0.0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      w[c] = c < nvalid[k] ? wsrc[k][c] : 0.f;
      maxabs = fmaxf(maxabs, fabsf(w[c]));
      acc = fma((double)w[c], (double)w[c], acc);
    }
    ww64[k] = acc;
    const int E = maxabs > 0.f ? ilogbf(maxabs) : 0;
    s2[k] = ldexp(1.0, -2 * E);
    float a = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const float v = scalbnf(w[c], -E);
      wd[k][c] = make_float2(v, v);
      a = fmaf(v, v, a);
    }
    ww32[k] = a;
    BlockSlot<P>& sl = slots[2 * tid + k];
    sl.seed = 1;
    sl.e = 15;
#pragma unroll
    for (int p = 0; p < P; ++p) sl.q[p] = 0;
    sl.ww = acc;
    sl.wsrc = wsrc[k];
    sl.nvalid = nvalid[k];
    if (nvalid[k] == 0 || acc == 0.0 || !isfinite(acc)) {
      // Nothing to search: an all-zero block's canonical fit is seed 1,
      // e = 15, q = 0 with error 0 (every candidate ties at 0).
      sl.err = acc;
      thr[k] = -INFINITY;
    } else {
      sl.err = INFINITY;
      thr[k] = INFINITY;
    }
  }
  // (w0, w1) pairs: the third basis column of C = 8 meets both blocks in one FMA.
  float2 wp[C];
#pragma unroll
  for (int c = 0; c < C; ++c) wp[c] = make_float2(wd[0][c].x, wd[1][c].x);
  const bool live0 = thr[0] != -INFINITY, live1 = thr[1] != -INFINITY;
  const unsigned lanes_below = (1u << lane) - 1u;
  int queued = 0;  // entries in this warp's queue (warp-uniform)
  __syncwarp();    // the warp's slots are written

  for (int k = 0; k < kChunks; ++k) {
    cp_async_wait_all();
    __syncthreads();  // chunk k landed everywhere; chunk k - 1's buffer is free
    if (k + 1 < kChunks) load_chunk<C>(qbuf + ((k + 1) & 1) * kChunk * C, table, k + 1, tid);
    cp_async_commit();
    if (__all_sync(0xffffffffu, thr[0] == -INFINITY && thr[1] == -INFINITY)) continue;
    const float4* qc = qbuf + (k & 1) * kChunk * C;
    const int s_first = k * kChunk + 1;
    const int ns = min(kChunk, kNumSeeds + 1 - s_first);  // the last table row is padding
    for (int j0 = 0; j0 < kChunk; j0 += kGroup) {
      // Residuals of kGroup seeds, then one branch for the rare survivors.
      float r0[kGroup], r1[kGroup];
      bool any = false;
#pragma unroll
      for (int u = 0; u < kGroup; ++u) {
        const float4* qs = qc + (j0 + u) * C;
        if constexpr (P == 3) {
          float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0;
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const float4 q = qs[c];
            const float2 q01 = make_float2(q.x, q.y), q22 = make_float2(q.z, q.w);
            a0 = __ffma2_rn(q01, wd[0][c], a0);
            a1 = __ffma2_rn(q01, wd[1][c], a1);
            a2 = __ffma2_rn(q22, wp[c], a2);
          }
          r0[u] = fmaf(-a0.x, a0.x, fmaf(-a0.y, a0.y, fmaf(-a2.x, a2.x, ww32[0])));
          r1[u] = fmaf(-a1.x, a1.x, fmaf(-a1.y, a1.y, fmaf(-a2.y, a2.y, ww32[1])));
        } else {
          float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const float4 q = qs[c];
            const float2 q01 = make_float2(q.x, q.y), q23 = make_float2(q.z, q.w);
            a0 = __ffma2_rn(q01, wd[0][c], a0);
            a1 = __ffma2_rn(q23, wd[0][c], a1);
            a2 = __ffma2_rn(q01, wd[1][c], a2);
            a3 = __ffma2_rn(q23, wd[1][c], a3);
          }
          r0[u] = fmaf(-a0.x, a0.x, fmaf(-a0.y, a0.y, fmaf(-a1.x, a1.x, fmaf(-a1.y, a1.y, ww32[0]))));
          r1[u] = fmaf(-a2.x, a2.x, fmaf(-a2.y, a2.y, fmaf(-a3.x, a3.x, fmaf(-a3.y, a3.y, ww32[1]))));
        }
        // !(r > thr) keeps a NaN residual in play.
        any = any || !(r0[u] > thr[0]) || !(r1[u] > thr[1]);
      }
      if (__any_sync(0xffffffffu, any)) {
        // Queue the survivors seed by seed (ascending), scoring a batch
        // whenever 32 are waiting; the thresholds then come from the slots.
#pragma unroll
        for (int u = 0; u < kGroup; ++u) {
          const uint32_t seed = (uint32_t)(s_first + j0 + u);
          const bool in = j0 + u < ns;
          const bool want0 = in && live0 && !(r0[u] > thr[0]);
          const bool want1 = in && live1 && !(r1[u] > thr[1]);
          const unsigned m0 = __ballot_sync(0xffffffffu, want0);
          const unsigned m1 = __ballot_sync(0xffffffffu, want1);
          if (want0) wq->ent[queued + __popc(m0 & lanes_below)] = seed | ((uint32_t)lane << 16);
          queued += __popc(m0);
          if (want1)
            wq->ent[queued + __popc(m1 & lanes_below)] = seed | ((uint32_t)lane << 16) | (1u << 21);
          queued += __popc(m1);
          if (queued >= 32) {
            __syncwarp();
            queued = drain_queue<C, P>(wq, queued, 32, wslots, exact, lane);
            if (live0) thr[0] = prune_threshold(slots[2 * tid].err, ww64[0], s2[0]);
            if (live1) thr[1] = prune_threshold(slots[2 * tid + 1].err, ww64[1], s2[1]);
          }
        }
      }
    }
  }
  __syncwarp();
  drain_queue<C, P>(wq, queued, 1, wslots, exact, lane);
  cp_async_wait_all();
  if (!active) return;

#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int blk = b0 + k;
    if (blk >= nb) break;
    const BlockSlot<P>& best = slots[2 * tid + k];
    // The winner's error, computed directly.
    const uint64_t st = seed_stream(best.seed);
    const double inv = 1.0 / (double)(1 << best.e);
    double err = 0.0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      double what = 0.0;
#pragma unroll
      for (int p = 0; p < P; ++p) what = fma(basis_entry<C, P>(st, c, p), (double)best.q[p], what);
      const double wc = c < nvalid[k] ? (double)wsrc[k][c] : 0.0;
      const double d = wc - what * inv;
      err = fma(d, d, err);
    }
    uint32_t r = best.seed << 16;
#pragma unroll
    for (int p = 0; p < P; ++p) r |= ((uint32_t)best.q[p] & 15u) << (4 * p);
    if constexpr (C == 8) r |= (uint32_t)best.e << 12;
    if (SEEDLM_IN_BOUNDS(g_check_flag, row, rows) && SEEDLM_IN_BOUNDS(g_check_flag, blk, rec_pitch))
      rec[(size_t)row * rec_pitch + blk] = r;
    if (err_out && SEEDLM_IN_BOUNDS(g_check_flag, (size_t)row * nb + blk, (size_t)rows * nb))
      err_out[(size_t)row * nb + blk] = err;
  }
  if constexpr (C == 12) {
    // The pair's exponent byte: block b0 in the low nibble, b0 + 1 (or 0).
    uint32_t byte = (uint32_t)slots[2 * tid].e & 15u;
    if (b0 + 1 < nb) byte |= ((uint32_t)slots[2 * tid + 1].e & 15u) << 4;
    if (SEEDLM_IN_BOUNDS(g_check_flag, row, rows) && SEEDLM_IN_BOUNDS(g_check_flag, b0 >> 1, e_pitch))
      eplane[(size_t)row * e_pitch + (b0 >> 1)] = (uint8_t)byte;
  }
}

template <int C, int P>
int launch_encode_t(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                    uint8_t* eplane, double* err, cudaStream_t stream, const DeviceInfo& dev) {
  const long long ipr = (f.nb + 1) / 2;
  const long long items = ipr * f.rows;
  if (items == 0) return SEEDLM_OK;
  const long long grid = (items + kEncThreads - 1) / kEncThreads;
  if (grid > 0x7fffffffll) return SEEDLM_EUNSUPPORTED;
  const size_t smem = 2 * kChunk * C * sizeof(float4) + 2 * kEncThreads * sizeof(BlockSlot<P>) +
                      (kEncThreads / 32) * sizeof(WarpQueue);
  int rc = allow_max_smem((const void*)encode_kernel<C, P>, dev);
  if (rc) return rc;
  // The seed tables live for this call only (one stream-ordered allocation:
  // fp32 bases, then fp64 G and G^-1).
  const size_t basis_bytes = (size_t)kTableRows * C * sizeof(float4);
  const size_t exact_bytes = (size_t)kTableRows * SeedExact<P>::kDoubles * sizeof(double);
  unsigned char* tables = nullptr;
  if ((rc = record_cuda_error(cudaMallocAsync(reinterpret_cast<void**>(&tables),
                                              basis_bytes + exact_bytes, stream))))
    return rc;
  float4* table = reinterpret_cast<float4*>(tables);
  double* exact = reinterpret_cast<double*>(tables + basis_bytes);
  basis_table_kernel<C, P><<<kTableRows / 256, 256, 0, stream>>>(table, exact);
  count_launch();
  encode_kernel<C, P><<<(unsigned)grid, kEncThreads, smem, stream>>>(
      W, ldw, f.rows, f.cols, f.nb, f.rec_pitch, f.e_pitch, rec, eplane, err, items, table, exact);
  count_launch();
  rc = record_cuda_error(cudaGetLastError());
  const int rc_free = record_cuda_error(cudaFreeAsync(tables, stream));
  return rc ? rc : rc_free;
}

}  // namespace

int launch_encode(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                  uint8_t* eplane, double* err, cudaStream_t stream, const DeviceInfo& dev) {
  if (f.C == 8) return launch_encode_t<8, 3>(f, W, ldw, rec, eplane, err, stream, dev);
  return launch_encode_t<12, 4>(f, W, ldw, rec, eplane, err, stream, dev);
}

}  // namespace seedlm
