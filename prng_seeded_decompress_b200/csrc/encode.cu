// encode.cu -- the encoder side of the format: for every block of W, the
// seed, quantised coefficients and exponent that reconstruct it best.
//
// SeedLM (paperhub.cn review thread, authors' replies on the cost of
// parameter optimisation): each block is matched against every seed's
// pseudo-random matrix U(s) (C x P), the coefficients are fitted and
// quantised, and the seed with the smallest reconstruction error wins; the
// search is parallel over blocks and seeds.  The pages fix no exponent or
// rounding rule; the reading used throughout this library:
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
// One thread owns one block (C = 8) or the two blocks that share an exponent
// byte (C = 12).  A CTA walks all 65,535 seeds in chunks: for each chunk it
// first builds U, G and G^-1 of every seed in shared memory (from the same
// bit stream the decoder uses, seedlm_device.cuh; G is exact in fp64 because
// U's entries are k / 32768), then every thread scores its blocks against the
// chunk.  All search arithmetic is fp64 and uses the expansion
//   err = ||w||^2 - 2^(1-e) q.(U^T w) + 2^(-2e) q^T G q,
// so a candidate costs a handful of fp64 operations once U^T w and t* of the
// seed are known.  A seed whose least-squares residual ||w||^2 - (U^T w).t*
// (a lower bound on every quantised candidate's error) already exceeds the
// best error found is skipped without scoring its exponents.  The winner's
// error is recomputed directly at the end.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

SEEDLM_CHECK_FLAG(encode)

namespace {

constexpr int kEncThreads = 128;
constexpr int kSeedChunk = 32;
constexpr int kNumSeeds = 65535;

template <int C, int P>
struct EncChunk {
  double U[kSeedChunk][C * P];  // U[c][p] at c * P + p
  double G[kSeedChunk][P * P];
  double Gi[kSeedChunk][P * P];
};

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

// In-place inverse of a symmetric positive definite P x P matrix by
// Gauss-Jordan elimination (no pivoting needed for SPD).
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

template <int C, int P>
__device__ void build_seed(EncChunk<C, P>& ch, int j, uint32_t seed) {
  const uint64_t st = seed_stream(seed);
  double u[C][P];
#pragma unroll
  for (int c = 0; c < C; ++c)
#pragma unroll
    for (int p = 0; p < P; ++p) {
      u[c][p] = basis_entry<C, P>(st, c, p);
      ch.U[j][c * P + p] = u[c][p];
    }
  double g[P * P];
#pragma unroll
  for (int p = 0; p < P; ++p)
#pragma unroll
    for (int r = 0; r < P; ++r) {
      double acc = 0.0;
#pragma unroll
      for (int c = 0; c < C; ++c) acc = fma(u[c][p], u[c][r], acc);  // exact
      g[p * P + r] = acc;
      ch.G[j][p * P + r] = acc;
    }
  spd_inverse<P>(g, ch.Gi[j]);
}

template <int P>
struct Best {
  double err;
  uint32_t seed;
  int e;
  int q[P];
};

template <int C, int P, int NBLK>
__global__ void __launch_bounds__(kEncThreads)
encode_kernel(const float* __restrict__ W, int64_t ldw, int rows, int cols, int nb,
              int rec_pitch, int e_pitch, uint32_t* __restrict__ rec,
              uint8_t* __restrict__ eplane, double* __restrict__ err_out, long long n_items) {
  __shared__ EncChunk<C, P> ch;
  const int ipr = (nb + NBLK - 1) / NBLK;  // items per row
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool active = item < n_items;
  const int row = active ? (int)(item / ipr) : 0;
  const int b0 = active ? (int)(item - (long long)row * ipr) * NBLK : 0;

  double w[NBLK][C];
  double ww[NBLK];
  Best<P> best[NBLK];
#pragma unroll
  for (int k = 0; k < NBLK; ++k) {
    ww[k] = 0.0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int col = (b0 + k) * C + c;
      const bool in = active && b0 + k < nb && col < cols &&
                      SEEDLM_IN_BOUNDS(g_check_flag, (size_t)row * ldw + col,
                                       (size_t)(rows - 1) * ldw + cols);
      w[k][c] = in ? (double)W[(size_t)row * ldw + col] : 0.0;
      ww[k] = fma(w[k][c], w[k][c], ww[k]);
    }
    best[k].err = __longlong_as_double(0x7ff0000000000000ll);  // +inf
    best[k].seed = 1;
    best[k].e = 15;
#pragma unroll
    for (int p = 0; p < P; ++p) best[k].q[p] = 0;
  }

  for (int s0 = 1; s0 <= kNumSeeds; s0 += kSeedChunk) {
    const int ns = min(kSeedChunk, kNumSeeds + 1 - s0);
    __syncthreads();  // the previous chunk is no longer read
    if (threadIdx.x < ns) build_seed<C, P>(ch, threadIdx.x, (uint32_t)(s0 + threadIdx.x));
    __syncthreads();
    for (int j = 0; j < ns; ++j) {
      const uint32_t seed = (uint32_t)(s0 + j);
#pragma unroll
      for (int k = 0; k < NBLK; ++k) {
        double b[P];
#pragma unroll
        for (int p = 0; p < P; ++p) {
          double acc = 0.0;
#pragma unroll
          for (int c = 0; c < C; ++c) acc = fma(ch.U[j][c * P + p], w[k][c], acc);
          b[p] = acc;
        }
        double t[P];
        double bt = 0.0;
#pragma unroll
        for (int p = 0; p < P; ++p) {
          double acc = 0.0;
#pragma unroll
          for (int r = 0; r < P; ++r) acc = fma(ch.Gi[j][p * P + r], b[r], acc);
          t[p] = acc;
          bt = fma(b[p], acc, bt);
        }
        // No quantised candidate of this seed beats its least-squares
        // residual ||w||^2 - b.t*; once that is above the best error so far
        // (beyond fp64 rounding), the seed's exponents need no scoring.
        if (ww[k] - bt > best[k].err + 1e-13 * ww[k]) continue;
        // Exponents in descending order: on an exact tie the larger e, met
        // first, stays.  |t* 2^e| shrinks with e, so once every q rounds to
        // 0 all smaller exponents give that same candidate (error ||w||^2,
        // met later): the loop ends there.
#pragma unroll 4
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
            double row = 0.5 * ch.G[j][p * P + p] * q[p];
#pragma unroll
            for (int r = p + 1; r < P; ++r) row = fma(ch.G[j][p * P + r], q[r], row);
            qgq = fma(q[p], row, qgq);
          }
          const double err = fma(2.0 * inv * inv, qgq, fma(-2.0 * inv, qb, ww[k]));
          if (err < best[k].err) {
            best[k].err = err;
            best[k].seed = seed;
            best[k].e = e;
#pragma unroll
            for (int p = 0; p < P; ++p) best[k].q[p] = (int)q[p];
          }
          if (zero) break;
        }
      }
    }
  }
  if (!active) return;

#pragma unroll
  for (int k = 0; k < NBLK; ++k) {
    const int blk = b0 + k;
    if (blk >= nb) break;
    // The winner's error, computed directly.
    const uint64_t st = seed_stream(best[k].seed);
    const double inv = 1.0 / (double)(1 << best[k].e);
    double err = 0.0;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      double what = 0.0;
#pragma unroll
      for (int p = 0; p < P; ++p) what = fma(basis_entry<C, P>(st, c, p), (double)best[k].q[p], what);
      const double d = w[k][c] - what * inv;
      err = fma(d, d, err);
    }
    uint32_t r = best[k].seed << 16;
#pragma unroll
    for (int p = 0; p < P; ++p) r |= ((uint32_t)best[k].q[p] & 15u) << (4 * p);
    if constexpr (C == 8) r |= (uint32_t)best[k].e << 12;
    if (SEEDLM_IN_BOUNDS(g_check_flag, row, rows) && SEEDLM_IN_BOUNDS(g_check_flag, blk, rec_pitch))
      rec[(size_t)row * rec_pitch + blk] = r;
    if (err_out && SEEDLM_IN_BOUNDS(g_check_flag, (size_t)row * nb + blk, (size_t)rows * nb))
      err_out[(size_t)row * nb + blk] = err;
  }
  if constexpr (C == 12) {
    // The pair's exponent byte: block b0 in the low nibble, b0 + 1 (or 0).
    uint32_t byte = (uint32_t)best[0].e & 15u;
    if (b0 + 1 < nb) byte |= ((uint32_t)best[1].e & 15u) << 4;
    if (SEEDLM_IN_BOUNDS(g_check_flag, row, rows) && SEEDLM_IN_BOUNDS(g_check_flag, b0 >> 1, e_pitch))
      eplane[(size_t)row * e_pitch + (b0 >> 1)] = (uint8_t)byte;
  }
}

template <int C, int P, int NBLK>
int launch_encode_t(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                    uint8_t* eplane, double* err, cudaStream_t stream) {
  const long long ipr = (f.nb + NBLK - 1) / NBLK;
  const long long items = ipr * f.rows;
  const long long grid = (items + kEncThreads - 1) / kEncThreads;
  if (grid > 0x7fffffffll) return SEEDLM_EUNSUPPORTED;
  encode_kernel<C, P, NBLK><<<(unsigned)grid, kEncThreads, 0, stream>>>(
      W, ldw, f.rows, f.cols, f.nb, f.rec_pitch, f.e_pitch, rec, eplane, err, items);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace

int launch_encode(const seedlm_format& f, const float* W, int64_t ldw, uint32_t* rec,
                  uint8_t* eplane, double* err, cudaStream_t stream) {
  if (f.C == 8) return launch_encode_t<8, 3, 1>(f, W, ldw, rec, eplane, err, stream);
  return launch_encode_t<12, 4, 2>(f, W, ldw, rec, eplane, err, stream);
}

}  // namespace seedlm
