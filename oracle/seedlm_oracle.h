/*
 * seedlm_oracle.h -- CPU oracle for SeedLM weight reconstruction and the
 * products that consume it.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
 * in __graft_entry__.py and the CPU-baseline leg of bench.py may load it.  It
 * shares no code, header, table or helper with the CUDA library; neither side
 * includes or links the other.
 *
 * What it computes (SeedLM: Compressing LLM Weights into Seeds of
 * Pseudo-Random Generators -- abstract, paperdance.org card): each block of C
 * weights is stored as a seed; the seed drives a linear feedback shift register
 * (LFSR) whose states fill a C x P matrix U; U is combined linearly with P
 * compressed coefficients t to give the block back, W_blk = U t (the review
 * thread on paperhub.cn names U and t the compression matrices of Eq (1)).
 * The coefficients are 4-bit integers q with a 4-bit exponent e shared by the
 * block, t = q * 2^-e (the same thread, authors' reply on data formats with
 * shared exponents; atlas.scime.ai summary, "Approach": only the seed and
 * the 4-bit coefficients are kept per block).  At inference the weights are rebuilt
 * on the fly and then multiplied with the activations (paperhub.cn thread,
 * authors' reply on how inference uses Eq (1)).
 *
 * Concrete parameters the pages leave open, fixed as the workload
 * specification fixes them:
 *   K = 16, Fibonacci LFSR with taps 16,14,13,11:
 *       bit = (s ^ s>>2 ^ s>>3 ^ s>>5) & 1 ;  s = (s >> 1) | (bit << 15)
 *   state_0 = seed;  U[c][p] = (state_{p*C + c} - 32768) / 32768.
 *   t_p = q_p * 2^-e, q_p two's-complement 4-bit, e unsigned 4-bit.
 *
 * Record layout (a reading; the pages give no bit order).  One uint32 per
 * block, blocks of a row in column order, row r starting at rec + r*rec_pitch:
 *   bits [16,32): seed;  bits [4p, 4p+4): q_p for p < P (LSB first);
 *   if P <= 3 the exponent sits in bits [4P, 4P+4) of the record;
 *   if P == 4 it sits in a separate nibble plane, row r at eplane + r*e_pitch,
 *   block b in byte b/2, low nibble for even b.
 * The last block of a row may run past `cols`; its extra weights are dropped.
 */
#ifndef SEEDLM_ORACLE_H
#define SEEDLM_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t C, P, K;       /* block length, latent dimension, seed bits (16) */
  int32_t rows, cols;    /* W is rows x cols */
  int32_t nb;            /* blocks per row = ceil(cols / C) */
  int32_t rec_pitch;     /* uint32 records between consecutive rows, >= nb */
  int32_t e_pitch;       /* bytes between rows of the exponent plane (P == 4) */
} oracle_format;

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)

/* One LFSR step. */
uint16_t oracle_lfsr_next(uint16_t s);

/* out[k] = state_k for k < n, state_0 = seed. */
void oracle_lfsr_states(uint16_t seed, int n, uint16_t* out);

/* Checks the fields of f; ORACLE_OK or ORACLE_EINVAL. */
int oracle_check_format(const oracle_format* f);

/* Decodes block b of row r: seed, q[0..P-1] (signed), e. */
int oracle_block_fields(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                        int r, int b, uint16_t* seed, int* q, int* e);

/* U(seed) as a C x P row-major array of doubles: U[c*P + p]. */
void oracle_block_basis(uint16_t seed, int C, int P, double* U);

/* U(seed) for every seed 1..65535, seed s at U_all + (s-1)*C*P. */
void oracle_basis_all(int C, int P, double* U_all);

/* Design-space variants (the pages' discussion of seed bit-width, block size
 * and latent dimension; review thread on paperhub.cn and the atlas.scime.ai
 * summary, "Limitations"): a K-bit Fibonacci register, 2 <= K <= 24, that
 * shifts right and feeds the parity of the tapped bits in at the top:
 *     bit = parity(s & taps);  s <- (s >> 1) | (bit << (K - 1)).
 * For K = 16 and taps = 0x2D this is the register above. */
uint32_t oracle_lfsr_next_k(uint32_t s, int K, uint32_t taps);

/* Steps from state 1 until the register first returns to 1; 0 if it has not
 * returned after 2^K steps (the taps are then not invertible). */
uint64_t oracle_lfsr_period_k(int K, uint32_t taps);

/* U(seed), C x P row-major, for a K-bit register: column p holds states
 * p*C .. p*C + C - 1 (state_0 = seed), each mapped to
 * (state - 2^(K-1)) / 2^(K-1). */
void oracle_block_basis_k(uint32_t seed, int C, int P, int K, uint32_t taps, double* U);

/* U(s) for every seed 1 .. 2^K - 1, seed s at U_all + (s-1)*C*P. */
void oracle_basis_all_k(int C, int P, int K, uint32_t taps, double* U_all);

/* W_blk = U t for block b of row r (all C weights, including any past cols). */
int oracle_reconstruct_block(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                             int r, int b, double* wblk);

/* W (rows x cols, row-major) in double; every entry is exact. */
int oracle_decompress(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                      double* W);

/* y[r] = sum_j W[r][j] x[j] in double; yabs[r] = sum_j |W[r][j]| |x[j]| if
 * yabs != NULL.  Rows are split over nthreads host threads (1 = serial). */
int oracle_gemv(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                const double* x, double* y, double* yabs, int nthreads);

/* Y[m][r] = sum_j W[r][j] X[m][j] for m < M (X is M x cols, Y is M x rows,
 * both row-major); Yabs likewise with absolute values, if not NULL. */
int oracle_gemm(const oracle_format* f, const uint32_t* rec, const uint8_t* eplane,
                const double* X, int M, double* Y, double* Yabs, int nthreads);

#ifdef __cplusplus
}
#endif

#endif /* SEEDLM_ORACLE_H */
