/*
 * seedlm_oracle.c -- plain, slow, obviously correct CPU oracle.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE (see seedlm_oracle.h).  Every function
 * follows the definition it cites, in that definition's order, in double
 * precision, with no blocking, fusion or reordering.  All reconstructed
 * weights are short dyadic rationals (an integer below 2^20 times 2^-(15+e)),
 * so every W value below is exact in double.
 */
#include "seedlm_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* LFSR step.  SeedLM abstract (paperdance.org card): the seed is fed into a
 * linear feedback shift register.  The 16-bit Fibonacci register with taps
 * 16,14,13,11 is the workload's choice; the pages name no polynomial. */
uint16_t oracle_lfsr_next(uint16_t s) {
  unsigned bit = ((unsigned)s ^ ((unsigned)s >> 2) ^ ((unsigned)s >> 3) ^ ((unsigned)s >> 5)) & 1u;
  return (uint16_t)(((unsigned)s >> 1) | (bit << 15));
}

/* state_0 is the seed itself; state_{k+1} = next(state_k). */
void oracle_lfsr_states(uint16_t seed, int n, uint16_t* out) {
  uint16_t s = seed;
  for (int k = 0; k < n; ++k) {
    out[k] = s;
    s = oracle_lfsr_next(s);
  }
}

int oracle_check_format(const oracle_format* f) {
  if (!f) return ORACLE_EINVAL;
  if (f->K != 16) return ORACLE_EINVAL;
  if (f->C < 1 || f->P < 1 || f->P > 4) return ORACLE_EINVAL;
  if (f->rows < 0 || f->cols < 0) return ORACLE_EINVAL;
  if (f->nb != (f->cols + f->C - 1) / f->C) return ORACLE_EINVAL;
  if (f->rec_pitch < f->nb) return ORACLE_EINVAL;
  if (f->P == 4 && f->e_pitch < (f->nb + 1) / 2) return ORACLE_EINVAL;
  return ORACLE_OK;
}

/* Two's-complement value of a 4-bit field. */
static int signed_nibble(unsigned v) { return (v & 8u) ? (int)v - 16 : (int)v; }

/* Record decoding, as laid out in seedlm_oracle.h. */
int oracle_block_fields(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                        int r, int b, uint16_t* seed, int* q, int* e) {
  uint32_t word = rec[(size_t)r * (size_t)f->rec_pitch + (size_t)b];
  *seed = (uint16_t)(word >> 16);
  for (int p = 0; p < f->P; ++p) q[p] = signed_nibble((word >> (4 * p)) & 15u);
  if (f->P <= 3) {
    *e = (int)((word >> (4 * f->P)) & 15u);
  } else {
    uint8_t byte = eplane[(size_t)r * (size_t)f->e_pitch + (size_t)(b / 2)];
    *e = (b % 2 == 0) ? (byte & 15) : (byte >> 4);
  }
  return ORACLE_OK;
}

/* U(seed), C x P: column p holds states p*C .. p*C + C - 1, each mapped to
 * (state - 32768) / 32768.  SeedLM abstract: the LFSR generates a random
 * matrix; atlas.scime.ai "Approach": a block is a linear combination of P
 * columns of that pseudo-random matrix. */
void oracle_block_basis(uint16_t seed, int C, int P, double* U) {
  uint16_t* st = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(C * P));
  oracle_lfsr_states(seed, C * P, st);
  for (int c = 0; c < C; ++c)
    for (int p = 0; p < P; ++p)
      U[c * P + p] = ((double)st[p * C + c] - 32768.0) / 32768.0;
  free(st);
}

void oracle_basis_all(int C, int P, double* U_all) {
  for (int s = 1; s <= 65535; ++s)
    oracle_block_basis((uint16_t)s, C, P, U_all + (size_t)(s - 1) * (size_t)(C * P));
}

/* The general register of seedlm_oracle.h, one step. */
uint32_t oracle_lfsr_next_k(uint32_t s, int K, uint32_t taps) {
  uint32_t v = s & taps, parity = 0;
  while (v) {
    parity ^= v & 1u;
    v >>= 1;
  }
  return (s >> 1) | (parity << (K - 1));
}

uint64_t oracle_lfsr_period_k(int K, uint32_t taps) {
  const uint64_t limit = (uint64_t)1 << K;
  uint32_t s = 1;
  for (uint64_t n = 1; n <= limit; ++n) {
    s = oracle_lfsr_next_k(s, K, taps);
    if (s == 1) return n;
  }
  return 0;
}

void oracle_block_basis_k(uint32_t seed, int C, int P, int K, uint32_t taps, double* U) {
  uint32_t* st = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)(C * P));
  uint32_t s = seed;
  for (int k = 0; k < C * P; ++k) {
    st[k] = s;
    s = oracle_lfsr_next_k(s, K, taps);
  }
  const double half = ldexp(1.0, K - 1);
  for (int c = 0; c < C; ++c)
    for (int p = 0; p < P; ++p) U[c * P + p] = ((double)st[p * C + c] - half) / half;
  free(st);
}

void oracle_basis_all_k(int C, int P, int K, uint32_t taps, double* U_all) {
  const uint32_t n = (1u << K) - 1u;
  for (uint32_t s = 1; s <= n; ++s)
    oracle_block_basis_k(s, C, P, K, taps, U_all + (size_t)(s - 1) * (size_t)(C * P));
}

/* Eq (1) of the paperhub.cn thread: W_blk = U t, with t_p = q_p * 2^-e. */
int oracle_reconstruct_block(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                             int r, int b, double* wblk) {
  uint16_t seed;
  int q[4], e;
  oracle_block_fields(f, rec, eplane, r, b, &seed, q, &e);
  double t[4];
  for (int p = 0; p < f->P; ++p) t[p] = ldexp((double)q[p], -e);
  double* U = (double*)malloc(sizeof(double) * (size_t)(f->C * f->P));
  oracle_block_basis(seed, f->C, f->P, U);
  for (int c = 0; c < f->C; ++c) {
    double acc = 0.0;
    for (int p = 0; p < f->P; ++p) acc += U[c * f->P + p] * t[p];
    wblk[c] = acc;
  }
  free(U);
  return ORACLE_OK;
}

int oracle_decompress(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                      double* W) {
  if (oracle_check_format(f) != ORACLE_OK) return ORACLE_EINVAL;
  double* wblk = (double*)malloc(sizeof(double) * (size_t)f->C);
  for (int r = 0; r < f->rows; ++r) {
    for (int b = 0; b < f->nb; ++b) {
      oracle_reconstruct_block(f, rec, eplane, r, b, wblk);
      for (int c = 0; c < f->C; ++c) {
        int j = b * f->C + c;
        if (j < f->cols) W[(size_t)r * (size_t)f->cols + (size_t)j] = wblk[c];
      }
    }
  }
  free(wblk);
  return ORACLE_OK;
}

/* Reconstruct-then-multiply (paperhub.cn thread, authors' reply on inference:
 * the weights are rebuilt from s and t and then used to compute the
 * activations): for each output m, r the plain sum over j of W[r][j] X[m][j]
 * in double, j in increasing order. */
typedef struct {
  const oracle_format* f;
  const uint32_t* rec;
  const uint8_t* eplane;
  const double* X;
  int M;
  double* Y;
  double* Yabs;
  int r0, r1;
} oracle_job;

static void* oracle_rows(void* arg) {
  oracle_job* jb = (oracle_job*)arg;
  const oracle_format* f = jb->f;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)(f->nb * f->C + 1));
  for (int r = jb->r0; r < jb->r1; ++r) {
    for (int b = 0; b < f->nb; ++b)
      oracle_reconstruct_block(f, jb->rec, jb->eplane, r, b, wrow + (size_t)b * (size_t)f->C);
    for (int m = 0; m < jb->M; ++m) {
      const double* x = jb->X + (size_t)m * (size_t)f->cols;
      double acc = 0.0, acc_abs = 0.0;
      for (int j = 0; j < f->cols; ++j) {
        acc += wrow[j] * x[j];
        acc_abs += fabs(wrow[j]) * fabs(x[j]);
      }
      jb->Y[(size_t)m * (size_t)f->rows + (size_t)r] = acc;
      if (jb->Yabs) jb->Yabs[(size_t)m * (size_t)f->rows + (size_t)r] = acc_abs;
    }
  }
  free(wrow);
  return NULL;
}

int oracle_gemm(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                const double* X, int M, double* Y, double* Yabs, int nthreads) {
  if (oracle_check_format(f) != ORACLE_OK || M < 0) return ORACLE_EINVAL;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > f->rows) nthreads = f->rows > 0 ? f->rows : 1;
  oracle_job* jobs = (oracle_job*)calloc((size_t)nthreads, sizeof(oracle_job));
  pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = (oracle_job){f, rec, eplane, X, M, Y, Yabs,
                           (int)((long long)f->rows * t / nthreads),
                           (int)((long long)f->rows * (t + 1) / nthreads)};
  }
  if (nthreads == 1) {
    oracle_rows(&jobs[0]);
  } else {
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, oracle_rows, &jobs[t]);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  }
  free(th);
  free(jobs);
  return ORACLE_OK;
}

int oracle_gemv(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                const double* x, double* y, double* yabs, int nthreads) {
  return oracle_gemm(f, rec, eplane, x, 1, y, yabs, nthreads);
}
