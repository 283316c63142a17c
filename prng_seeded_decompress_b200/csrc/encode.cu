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
// Two kernels.  seed_table_kernel computes, once per call and for every seed,
// G (exact in fp64: U's entries are k / 32768) and G^-1, and an orthonormal
// basis Q(s) of U(s)'s column space (Gram-Schmidt in fp64, each column
// orthogonalised twice), stored as the B operand of the tensor-core filter.
//
// encode_tc_kernel: a least-squares filter on the tensor cores, then exact
// scoring of the few seeds it cannot rule out.  For every block and seed the
// residual r(s) = ||w||^2 - ||Q(s)^T w||^2 is a lower bound on the error of
// every quantised candidate of that seed; only a seed whose residual is not
// above the block's best error so far plus a margin is scored exactly
// (seed_candidate: fp64, t* = G^-1 U^T w, the exponents in descending order
// with err = ||w||^2 - 2^(1-e) q.(U^T w) + 2^(-2e) q^T G q).  On Gaussian
// blocks about 3 in 10^4 seeds get that far.  The projections Q(s)^T w come
// from tcgen05 MMAs (description at the kernel); the exact scoring runs in
// warp-wide batches.
//
// The filter never changes the result: a seed is skipped only when its
// residual, computed within a proven error bound, exceeds the best error by
// more than that bound, so none of its candidates can reach the best error
// (candidates replace the best only on a strictly smaller error).  The
// winner's error is recomputed directly at the end.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"
#include "tcgen05.cuh"

namespace seedlm {

SEEDLM_CHECK_FLAG(encode)

// Set when a bounded wait of the search gave up.
__device__ unsigned int g_enc_error = 0;

namespace {

constexpr int kNumSeeds = 65535;
constexpr int kTableRows = 65536;  // exact-table rows: row i holds seed i + 1
constexpr double kPruneMargin = 2e-4;  // relative to ||w||^2, ten times the filter's error bound
constexpr uint64_t kEncWaitLimit = 2000000000ull;  // ns a hand-over wait may take

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
// whose residual exceeds it cannot beat the best error.  Once the best error
// is 0 nothing can (strict <).
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
// a time with every lane busy.  Entry: seed | lane << 16 (the block of that
// lane).
constexpr int kQueue = 64;  // < 32 left over + at most 32 added per seed
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
      const BlockSlot<P>& bs = wslots[(en >> 16) & 31u];
      const Cand cd = seed_candidate<C, P>(en & 0xffffu, bs.wsrc, bs.nvalid, bs.ww, exact);
      wq->err[lane] = cd.err;
      wq->eq[lane] = cd.eq;
    }
    __syncwarp();
    for (int i = 0; i < n; ++i) {
      const uint32_t en = wq->ent[base + i];
      if (((en >> 16) & 31u) == (uint32_t)lane) {
        BlockSlot<P>& bs = wslots[lane];
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

// ---------------------------------------------------------------- tensor-core filter
//
// The projections on the tensor cores: D[block][(p, s)] = sum_c w[c] Q(s)[c][p]
// for 128 blocks (the TMEM lanes) against 32 (C = 8) or 24 (C = 12) seeds at
// a time, kind::f16 with fp32 accumulation, every operand split exactly into
// an fp16 high part and an fp16 rest: D = A_hi B_hi + A_hi B_lo + A_lo B_hi.  For C = 8 the two B
// parts share one K = 16 row ([Q_hi | Q_lo] against [w_hi | w_hi] and
// [w_lo | 0]), so a stage is two MMAs; for C = 12 (K padded to 16) three.
// The block is scaled by 2^-E (exact) so that max|w| lies in [1, 2), and
// |Q| <= 1.  The dropped A_lo B_lo term and the fp16 rounding of the rests
// are below 2^-22 of each product (plus 2^-25 absolute, fp16's smallest
// step); the accumulation adds at most about 20 fp32 roundings of
// sum_c |w_c Q_cp| <= ||w||, so each coordinate is within 4e-6 ||w||, and
// with ||w||^2 in fp32 and the final subtraction the residual is within
// 2e-5 ||w||^2.  Q itself is orthonormal to fp64 rounding and spans U(s)'s
// column space to within kappa(U) 2^-53 < 1e-10 (kappa(U) < 4e5 over all
// seeds).  A seed is skipped when r > best + 2e-4 ||w||^2.
//
// Warps 0-3 (one TMEM lane quarter each, one block per thread) write A,
// read each stage's 96 accumulator columns and test the residuals
// against the threshold, queueing survivors for exact scoring; warp 4 issues
// the MMAs (one elected lane); warp 5 copies the B stages, precomputed in the
// MMA's shared-memory layout, with bulk copies.  All hand-overs are
// mbarriers with bounded waits: the epilogue spins (its hand-over comes every
// few hundred cycles), the MMA and copy warps park on suspend-hinted waits
// so that they leave the issue slots to the epilogue (measured: no loss).

template <int C>
struct TcEnc {
  static constexpr int P = (C == 8) ? 3 : 4;
  // Seeds per stage: N = 96 MMA columns either way, so the accumulators of
  // two stages (and A) fit in 256 TMEM columns and two CTAs share an SM.
  // (16 seeds per stage with 4 or 3 stages measured 15-25 % slower.)
  static constexpr int kSeeds = (C == 8) ? 32 : 24;
  static constexpr int kHalves = (kSeeds + 15) / 16;  // 16-seed halves of a stage
  static constexpr int kStages = (kNumSeeds + kSeeds - 1) / kSeeds;  // per sweep
  static constexpr int kRows = kStages * kSeeds;       // table rows incl. zero padding
  static constexpr int N = kSeeds * P;                 // MMA columns: (p, s), p-major
  // Seeds of the last stage that exist (the rest are padding rows).
  static constexpr int kLastSeeds = kNumSeeds - (kStages - 1) * kSeeds;
  static constexpr uint32_t kLastMask = (kLastSeeds == 32) ? 0xffffffffu : ((1u << kLastSeeds) - 1u);
  static constexpr int kPiecesB = (C == 8) ? 1 : 2;
  static constexpr int kSlabBytes = N * 16 * 2;        // one N x 16 fp16 operand
  static constexpr int kStageBytes = kSlabBytes * kPiecesB;
  static constexpr int kBS = (C == 8) ? 8 : 4;         // B stages in shared memory
  static constexpr int kDS = 2;                        // accumulator stages in TMEM
  static constexpr int kACols = 16;                    // A: two pieces of 8 columns
  static constexpr int kTmemCols = (kACols + kDS * N <= 256) ? 256 : 512;
  static constexpr int kCtasPerSm = 512 / kTmemCols;
  static_assert(kACols + kDS * N <= kTmemCols, "TMEM budget");
  static constexpr int kThreads = 6 * 32;
  static constexpr int kMmaWarp = 4, kLoaderWarp = 5;
  static_assert(N % 16 == 0 && N <= 256, "M = 128 MMA shape");
  // The epilogue reads whole 16-column halves: the last one may run past its
  // stage, never past the allocation.
  static_assert(kACols + (kDS - 1) * N + (P - 1) * kSeeds + 16 * kHalves <= kTmemCols,
                "TMEM reads stay inside the allocation");
};

// Byte offset of element (n, k) in an N x 16 fp16 operand, K-major core
// matrices (8 rows x 16 bytes; K neighbours 128 B apart, 8-row groups 256 B).
__host__ __device__ constexpr int slab16_byte(int n, int k) {
  return (n >> 3) * 256 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

// Row i of the tables (seed i + 1): G = U^T U and G^-1 for exact scoring,
// and the orthonormal basis split into fp16 high parts and rests at
// (n = p * kSeeds + s, k) of its stage's B operand(s).
template <int C, int P>
__global__ void __launch_bounds__(256) seed_table_kernel(unsigned char* __restrict__ btab,
                                                         double* __restrict__ exact) {
  using T = TcEnc<C>;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T::kRows) return;
  unsigned char* stage = btab + (size_t)(i / T::kSeeds) * T::kStageBytes;
  const int s = i % T::kSeeds;
  double q[C][P];
  if (i < kNumSeeds) {
    const uint64_t st = seed_stream((uint32_t)(i + 1));
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
    // Gram-Schmidt, each column orthogonalised twice against the previous ones.
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
  } else {
#pragma unroll
    for (int c = 0; c < C; ++c)
#pragma unroll
      for (int p = 0; p < P; ++p) q[c][p] = 0.0;
  }
#pragma unroll
  for (int p = 0; p < P; ++p) {
    const int n = p * T::kSeeds + s;
    __half hi[16], lo[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) hi[k] = lo[k] = __float2half_rn(0.f);
#pragma unroll
    for (int c = 0; c < C; ++c) {
      hi[c] = __double2half(q[c][p]);
      lo[c] = __double2half(q[c][p] - (double)__half2float(hi[c]));
    }
    if constexpr (C == 8) {
      // One operand: k < 8 the high parts, k >= 8 the rests.
#pragma unroll
      for (int k = 0; k < 16; ++k)
        *reinterpret_cast<__half*>(stage + slab16_byte(n, k)) = (k < 8) ? hi[k] : lo[k - 8];
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        *reinterpret_cast<__half*>(stage + slab16_byte(n, k)) = hi[k];
        *reinterpret_cast<__half*>(stage + T::kSlabBytes + slab16_byte(n, k)) = lo[k];
      }
    }
  }
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

template <int C, int P>
__global__ void __launch_bounds__(TcEnc<C>::kThreads, TcEnc<C>::kCtasPerSm)
encode_tc_kernel(const float* __restrict__ W, int64_t ldw, int rows, int cols, int nb,
                 int rec_pitch, int e_pitch, uint32_t* __restrict__ rec,
                 uint8_t* __restrict__ eplane, double* __restrict__ err_out, long long n_items,
                 int tiles, const unsigned char* __restrict__ btab,
                 const double* __restrict__ exact) {
  using T = TcEnc<C>;
  constexpr int BS = T::kBS, DS = T::kDS, N = T::N;
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* bring = smem;  // [BS][kStageBytes]
  BlockSlot<P>* slots = reinterpret_cast<BlockSlot<P>*>(smem + BS * T::kStageBytes);  // [128]
  WarpQueue* queues = reinterpret_cast<WarpQueue*>(slots + 128);                      // [4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(queues + 4);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2 * BS + 2 * DS + 1);  // TMEM base, abort
  const uint32_t bar0 = tc::smem_u32(bars);
  auto bfull = [&](int b) { return bar0 + 8 * b; };
  auto bempty = [&](int b) { return bar0 + 8 * (BS + b); };
  auto dfull = [&](int d) { return bar0 + 8 * (2 * BS + d); };
  auto dempty = [&](int d) { return bar0 + 8 * (2 * BS + DS + d); };
  const uint32_t afull = bar0 + 8 * (2 * BS + 2 * DS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (!SEEDLM_IN_BOUNDS(g_check_flag,
                        (size_t)(reinterpret_cast<unsigned char*>(tslot + 2) - smem) - 1,
                        seedlm_dynamic_smem_bytes()))
    return;
  if (tid == 0) {
    for (int b = 0; b < BS; ++b) {
      tc::mbar_init(bfull(b), 1);
      tc::mbar_init(bempty(b), 1);
    }
    for (int d = 0; d < DS; ++d) {
      tc::mbar_init(dfull(d), 1);
      tc::mbar_init(dempty(d), 4);
    }
    tc::mbar_init(afull, 4);
    tc::fence_mbar_init();
    tslot[1] = 0u;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(tslot), T::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tslot[0];
  volatile uint32_t* abort_flag = tslot + 1;
  bool ok = true;
  const int my_tiles = tiles > (int)blockIdx.x ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = my_tiles * T::kStages;  // stages this CTA runs

  if (warp == T::kLoaderWarp) {
    if (lane == 0) {
      for (int gs = 0; gs < total; ++gs) {
        const int b = gs % BS, g = gs % T::kStages;
        if (gs >= BS) ok = tc::mbar_wait_or_abort(bempty(b), ((gs / BS) - 1) & 1, kEncWaitLimit, abort_flag) && ok;
        if (SEEDLM_IN_BOUNDS(g_check_flag, g, T::kStages)) {
          tc::mbar_arrive_expect_tx(bfull(b), T::kStageBytes);
          tc::bulk_g2s(tc::smem_u32(bring + b * T::kStageBytes), btab + (size_t)g * T::kStageBytes,
                       T::kStageBytes, bfull(b));
        } else {
          tc::mbar_arrive(bfull(b));
        }
      }
      // Every copy has landed before the CTA may exit.
      for (int k = 0; k < BS && k < total; ++k) {
        const int gs = total - 1 - k;
        ok = tc::mbar_wait(bfull(gs % BS), (gs / BS) & 1, kEncWaitLimit) && ok;
      }
    }
    __syncwarp();
  } else if (warp == T::kMmaWarp) {
    const uint32_t idesc = tc::idesc_f16(N, 0);
    for (int gs = 0; gs < total; ++gs) {
      const int b = gs % BS, d = gs % DS;
      if (gs % T::kStages == 0)  // a new tile: its A pieces are in TMEM
        ok = tc::mbar_wait_or_abort(afull, (gs / T::kStages) & 1, kEncWaitLimit, abort_flag) && ok;
      ok = tc::mbar_wait_or_abort(bfull(b), (gs / BS) & 1, kEncWaitLimit, abort_flag) && ok;
      if (gs >= DS) ok = tc::mbar_wait_or_abort(dempty(d), ((gs / DS) - 1) & 1, kEncWaitLimit, abort_flag) && ok;
      __syncwarp();
      tc::fence_after_sync();
      const uint32_t dt = tmem + T::kACols + d * N;
      const uint32_t sb = tc::smem_u32(bring + b * T::kStageBytes);
      const uint64_t bhi = tc::smem_desc(sb, 128, 256);
      if constexpr (C == 8) {
        tc::mma_f16_ts_warp(dt, tmem, bhi, idesc, 0u);      // [w_hi | w_hi] . [Q_hi | Q_lo]
        tc::mma_f16_ts_warp(dt, tmem + 8, bhi, idesc, 1u);  // [w_lo | 0] . [Q_hi | Q_lo]
      } else {
        const uint64_t blo = tc::smem_desc(sb + T::kSlabBytes, 128, 256);
        tc::mma_f16_ts_warp(dt, tmem, bhi, idesc, 0u);
        tc::mma_f16_ts_warp(dt, tmem, blo, idesc, 1u);
        tc::mma_f16_ts_warp(dt, tmem + 8, bhi, idesc, 1u);
      }
      tc::mma_commit_warp(bempty(b));
      tc::mma_commit_warp(dfull(d));
    }
    // The last commits have arrived before the CTA may exit.
    for (int k = 0; k < BS && k < total; ++k) {
      const int gs = total - 1 - k;
      ok = tc::mbar_wait(bempty(gs % BS), (gs / BS) & 1, kEncWaitLimit) && ok;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue: one block per thread
    const unsigned lanes_below = (1u << lane) - 1u;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    WarpQueue* wq = queues + warp;
    BlockSlot<P>* wslots = slots + 32 * warp;
    BlockSlot<P>& sl = slots[tid];
    const int ipr = (nb + 1) / 2;
    int gs = 0;
    for (int it = 0; it < my_tiles; ++it) {
      const int tile = (int)blockIdx.x + it * (int)gridDim.x;
      const long long item = (long long)tile * 64 + (tid >> 1);
      const int k = tid & 1;
      const bool active = item < n_items;
      const int row = active ? (int)(item / ipr) : 0;
      const int blk = active ? (int)(item - (long long)row * ipr) * 2 + k : 0;
      const bool valid = active && blk < nb;
      int nvalid = valid ? min(C, cols - blk * C) : 0;
      const float* wsrc = W + (size_t)row * ldw + (size_t)blk * C;
      if (nvalid > 0 &&
          !SEEDLM_IN_BOUNDS(g_check_flag, (size_t)row * ldw + (size_t)blk * C + nvalid - 1,
                            (size_t)(rows - 1) * ldw + cols))
        nvalid = 0;
      float w[C];
      float maxabs = 0.f;
      double ww64 = 0.0;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        w[c] = c < nvalid ? wsrc[c] : 0.f;
        maxabs = fmaxf(maxabs, fabsf(w[c]));
        ww64 = fma((double)w[c], (double)w[c], ww64);
      }
      const int E = maxabs > 0.f ? ilogbf(maxabs) : 0;
      const double s2 = ldexp(1.0, -2 * E);
      float ww32 = 0.f;
      __half hi[16], lo[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) hi[c] = lo[c] = __float2half_rn(0.f);
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const float v = scalbnf(w[c], -E);
        ww32 = fmaf(v, v, ww32);
        hi[c] = __float2half_rn(v);
        lo[c] = __float2half_rn(v - __half2float(hi[c]));
      }
      // A: columns 0-7 the high parts (C = 8: repeated at k = 8..15),
      // columns 8-15 the rests.
      uint32_t a[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        a[j] = (C == 8) ? pack_half2(hi[(2 * j) & 7], hi[(2 * j + 1) & 7])
                        : pack_half2(hi[2 * j], hi[2 * j + 1]);
        a[8 + j] = pack_half2(lo[2 * j], lo[2 * j + 1]);
      }
      tc::tmem_st16(tmem + lane_base, a);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(afull);

      sl.seed = 1;
      sl.e = 15;
#pragma unroll
      for (int p = 0; p < P; ++p) sl.q[p] = 0;
      sl.ww = ww64;
      sl.wsrc = wsrc;
      sl.nvalid = nvalid;
      const bool live = !(nvalid == 0 || ww64 == 0.0 || !isfinite(ww64));
      sl.err = live ? INFINITY : ww64;  // a dead block keeps seed 1, e = 15, q = 0
      float thr = live ? INFINITY : -INFINITY;
      float base = ww32 - thr;  // r' = base - sum of squares < 0  <=>  r < thr
      int queued = 0;
      __syncwarp();

      // Pipelined over half stages (16 seeds): the TMEM loads of the next
      // half are in flight while the current half is tested.
      auto dcol = [&](int dd, int p, int h) {
        // (a last half of fewer than 16 seeds reads columns of the next p or
        // stage as well: read, never used)
        return tmem + lane_base + T::kACols + dd * N + p * T::kSeeds + 16 * h;
      };
      // Halves of 16 seeds: the loads of the next half are in flight while
      // the current one is tested.  With one half per stage the stage loop
      // is unrolled by two so that the register buffer of every half is
      // known at compile time.
      constexpr int H = T::kHalves;
      constexpr int U = (H == 1) ? 2 : 1;
      static_assert(T::kStages % U == 0, "whole unrolled stage pairs");
      uint32_t vb[2][P][16];
      ok = tc::mbar_spin_or_abort(dfull(gs % DS), (gs / DS) & 1, kEncWaitLimit, abort_flag) && ok;
      __syncwarp();
      tc::fence_after_sync();
#pragma unroll
      for (int p = 0; p < P; ++p) tc::tmem_ld16_async(dcol(gs % DS, p, 0), vb[0][p]);
      for (int g0 = 0; g0 < T::kStages; g0 += U) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int g = g0 + u;
          const int d = gs % DS;
          float rp[H][16];
          uint32_t neg = 0;
#pragma unroll
          for (int h = 0; h < H; ++h) {
            const int b = (H == 1) ? u : h;  // buffer of this half
#pragma unroll
            for (int p = 0; p < P; ++p) tc::tmem_wait_ld_tie(vb[b][p]);
            if (h + 1 < H) {
#pragma unroll
              for (int p = 0; p < P; ++p) tc::tmem_ld16_async(dcol(d, p, h + 1), vb[1 - b][p]);
            } else {
              // The whole stage is in registers: release it and start the
              // next stage's loads.
              tc::fence_before_sync();
              __syncwarp();
              if (lane == 0) tc::mbar_arrive(dempty(d));
              if (g + 1 < T::kStages) {
                const int d2 = (gs + 1) % DS;
                ok = tc::mbar_spin_or_abort(dfull(d2), ((gs + 1) / DS) & 1, kEncWaitLimit, abort_flag) && ok;
                __syncwarp();
                tc::fence_after_sync();
#pragma unroll
                for (int p = 0; p < P; ++p) tc::tmem_ld16_async(dcol(d2, p, 0), vb[1 - b][p]);
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float2 r2 = make_float2(base, base);
#pragma unroll
              for (int p = 0; p < P; ++p) {
                const float2 x =
                    make_float2(__uint_as_float(vb[b][p][2 * j]), __uint_as_float(vb[b][p][2 * j + 1]));
                r2 = __ffma2_rn(make_float2(-x.x, -x.y), x, r2);
              }
              rp[h][2 * j] = r2.x;
              rp[h][2 * j + 1] = r2.y;
              if (16 * h + 2 * j < T::kSeeds) neg |= __float_as_uint(r2.x) | __float_as_uint(r2.y);
            }
          }
          if (__any_sync(0xffffffffu, live && (neg >> 31))) {
            // Queue this stage's survivors in seed order (tested against the
            // threshold the residuals were computed with: never tighter than
            // the current one), visiting only seeds some lane kept.
            uint32_t mine = 0;
#pragma unroll
            for (int h = 0; h < H; ++h)
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (16 * h + j < T::kSeeds) mine |= (__float_as_uint(rp[h][j]) >> 31) << (16 * h + j);
            if (!live) mine = 0;
            if (g == T::kStages - 1) mine &= T::kLastMask;  // padding rows are no seeds
            uint32_t todo = __reduce_or_sync(0xffffffffu, mine);
            while (todo) {
              const int j = __ffs(todo) - 1;
              todo &= todo - 1;
              const bool want = (mine >> j) & 1u;
              const unsigned m = __ballot_sync(0xffffffffu, want);
              if (want)
                wq->ent[queued + __popc(m & lanes_below)] =
                    (uint32_t)(g * T::kSeeds + j + 1) | ((uint32_t)lane << 16);
              queued += __popc(m);
              if (queued >= 32) {
                __syncwarp();
                queued = drain_queue<C, P>(wq, queued, 32, wslots, exact, lane);
                if (live) {
                  thr = prune_threshold(sl.err, ww64, s2);
                  base = ww32 - thr;
                }
              }
            }
          }
          ++gs;
        }
      }
      __syncwarp();
      drain_queue<C, P>(wq, queued, 1, wslots, exact, lane);

      // The block's record (and error), the winner's error computed directly.
      uint32_t e_me = (uint32_t)sl.e & 15u;
      if (valid) {
        const uint64_t st = seed_stream(sl.seed);
        const double inv = 1.0 / (double)(1 << sl.e);
        double err = 0.0;
#pragma unroll
        for (int c = 0; c < C; ++c) {
          double what = 0.0;
#pragma unroll
          for (int p = 0; p < P; ++p) what = fma(basis_entry<C, P>(st, c, p), (double)sl.q[p], what);
          const double wc = c < nvalid ? (double)wsrc[c] : 0.0;
          const double dd = wc - what * inv;
          err = fma(dd, dd, err);
        }
        uint32_t r = sl.seed << 16;
#pragma unroll
        for (int p = 0; p < P; ++p) r |= ((uint32_t)sl.q[p] & 15u) << (4 * p);
        if constexpr (C == 8) r |= (uint32_t)sl.e << 12;
        if (SEEDLM_IN_BOUNDS(g_check_flag, row, rows) && SEEDLM_IN_BOUNDS(g_check_flag, blk, rec_pitch))
          rec[(size_t)row * rec_pitch + blk] = r;
        if (err_out && SEEDLM_IN_BOUNDS(g_check_flag, (size_t)row * nb + blk, (size_t)rows * nb))
          err_out[(size_t)row * nb + blk] = err;
      } else {
        e_me = 0u;
      }
      if constexpr (C == 12) {
        // The pair's exponent byte: even lane (block 2j) low nibble, its
        // neighbour (block 2j + 1, or nothing) high nibble.
        const uint32_t e_hi = __shfl_down_sync(0xffffffffu, e_me, 1);
        if (k == 0 && valid &&
            SEEDLM_IN_BOUNDS(g_check_flag, row, rows) && SEEDLM_IN_BOUNDS(g_check_flag, blk >> 1, e_pitch))
          eplane[(size_t)row * e_pitch + (blk >> 1)] = (uint8_t)(e_me | (e_hi << 4));
      }
      __syncwarp();
    }
  }

  if (!ok) atomicOr(&g_enc_error, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, T::kTmemCols);
  }
}

template <int C, int P>
int launch_encode_t(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                    uint8_t* eplane, double* err, cudaStream_t stream, const DeviceInfo& dev) {
  using T = TcEnc<C>;
  const long long ipr = (f.nb + 1) / 2;
  const long long items = ipr * f.rows;
  if (items == 0) return SEEDLM_OK;
  const long long tiles = (items + 63) / 64;  // 128 blocks per tile
  if (tiles > 0x7fffffffll) return SEEDLM_EUNSUPPORTED;
  int rc = allow_max_smem((const void*)encode_tc_kernel<C, P>, dev);
  if (rc) return rc;
  // The seed tables live for this call only (one stream-ordered allocation:
  // fp64 G and G^-1, then the tensor-core B operands).
  const size_t exact_bytes = (size_t)kTableRows * SeedExact<P>::kDoubles * sizeof(double);
  const size_t btab_bytes = (size_t)T::kStages * T::kStageBytes;  // kRows seeds
  unsigned char* tables = nullptr;
  if ((rc = record_cuda_error(cudaMallocAsync(reinterpret_cast<void**>(&tables),
                                              exact_bytes + btab_bytes, stream))))
    return rc;
  double* exact = reinterpret_cast<double*>(tables);
  unsigned char* btab = tables + exact_bytes;
  seed_table_kernel<C, P><<<(T::kRows + 255) / 256, 256, 0, stream>>>(btab, exact);
  count_launch();
  const long long cap = (long long)dev.num_sms * T::kCtasPerSm;
  const int grid = (int)(tiles < cap ? tiles : cap);
  const size_t smem = (size_t)T::kBS * T::kStageBytes + 128 * sizeof(BlockSlot<P>) +
                      4 * sizeof(WarpQueue) + (2 * T::kBS + 2 * T::kDS + 1) * 8 + 8;
  encode_tc_kernel<C, P><<<grid, T::kThreads, smem, stream>>>(
      W, ldw, f.rows, f.cols, f.nb, f.rec_pitch, f.e_pitch, rec, eplane, err, items, (int)tiles,
      btab, exact);
  count_launch();
  rc = record_cuda_error(cudaGetLastError());
  const int rc_free = record_cuda_error(cudaFreeAsync(tables, stream));
  return rc ? rc : rc_free;
}

}  // namespace

int read_and_clear_encode_error(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, g_enc_error, sizeof(v));
  if (err == cudaSuccess && v) err = cudaMemcpyToSymbol(g_enc_error, &zero, sizeof(zero));
  *out = v;
  return record_cuda_error(err);
}

int launch_encode(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                  uint8_t* eplane, double* err, cudaStream_t stream, const DeviceInfo& dev) {
  if (f.C == 8) return launch_encode_t<8, 3>(f, W, ldw, rec, eplane, err, stream, dev);
  return launch_encode_t<12, 4>(f, W, ldw, rec, eplane, err, stream, dev);
}

}  // namespace seedlm
