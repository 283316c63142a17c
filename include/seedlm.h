/*
 * seedlm.h -- C ABI of libseedlm.so: SeedLM weight reconstruction fused with
 * the matrix-vector and small-batch matrix products that consume it, on B200
 * (sm_100a).
 *
 * The operation (SeedLM: Compressing LLM Weights into Seeds of Pseudo-Random
 * Generators -- abstract on the paperdance.org card; "Approach" on the
 * atlas.scime.ai summary): a weight matrix W (rows x cols) is cut along each
 * row into blocks of C weights.  Each block is stored as a 16-bit seed, P
 * signed 4-bit coefficients q_p and one 4-bit exponent e shared by the block.
 * The seed starts a 16-bit Fibonacci LFSR (taps 16,14,13,11):
 *     bit = (s ^ s>>2 ^ s>>3 ^ s>>5) & 1 ;  s <- (s >> 1) | (bit << 15)
 * with state_0 = seed; U is the C x P matrix U[c][p] = (state_{pC+c} - 32768)
 * / 32768, and the block is W_blk = U t with t_p = q_p 2^-e (Eq (1) as the
 * paperhub.cn review thread names it: U and t are the compression matrices).
 * At inference W is never stored: each call rebuilds the blocks on the fly and
 * consumes them at once (same thread, the authors' reply on how inference uses
 * s and t).  Every rebuilt weight is an integer below 2^20 times 2^-(15+e), so
 * it is exact in fp32.
 *
 * Supported formats: (C, P, K) = (8, 3, 16) -- 32 bits per 8 weights, 4 bits
 * per weight -- and (12, 4, 16) -- 36 bits per 12 weights, 3 bits per weight.
 *
 * Record layout (the pages give none; this is the library's reading):
 *   rec: one uint32 per block, blocks of a row in column order, row r at
 *        rec + r * rec_pitch.  bits [16,32) seed; bits [4p, 4p+4) q_p for
 *        p < P, two's complement.  (8,3): e in bits [12,16).
 *   eplane (only for (12,4)): the exponents, row r at eplane + r * e_pitch,
 *        block b in byte b/2, low nibble for even b.
 *   Blocks run along a row; the last block of a row may extend past `cols`,
 *   its weights beyond `cols` are dropped (as if x were zero-padded).
 *   Records between nb and rec_pitch are padding and are never used.
 *   A seed of 0 is accepted and gives the LFSR's fixed point (all states 0,
 *   U = -1 everywhere).
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers, unless a function says HOST.
 *     The caller owns every buffer.  No call allocates device memory except
 *     seedlm_encode, which takes its seed tables from the stream-ordered
 *     allocator for the duration of the call (seedlm_gemm_smallM_noalloc's
 *     scratch is an array inside the library image).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; the call returns once it is enqueued.
 *   - Return value 0 = success, negative = error (SEEDLM_E*), with no work
 *     enqueued when the arguments are rejected.  Nothing aborts or prints.
 *   - Alignment: rec must be 16-byte aligned (rec_pitch is a multiple of 4,
 *     so every row is); x and X 2-byte aligned; y, Y and W 4-byte aligned.
 *   - Results are fp32.  Decompression is bit-exact.  Products accumulate in
 *     fp32 in a fixed order per shape, so repeated calls give identical bits;
 *     the error against the exact product stays within 1e-5 * sum_j |W_rj x_j|
 *     for the shapes this library targets.
 */
#ifndef SEEDLM_H
#define SEEDLM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Only the functions below are exported from libseedlm.so. */
#if defined(__GNUC__)
#define SEEDLM_API __attribute__((visibility("default")))
#else
#define SEEDLM_API
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* seedlm_stream;

typedef struct seedlm_format {
  int32_t C, P, K;    /* (8,3,16) or (12,4,16); others -> SEEDLM_EUNSUPPORTED     */
  int32_t rows;       /* rows of W (outputs of the product), >= 0                 */
  int32_t cols;       /* cols of W (inputs of the product), >= 0                  */
  int32_t nb;         /* blocks per row; must equal ceil(cols / C)                */
  int32_t rec_pitch;  /* uint32 records from one row to the next: >= nb, % 4 == 0 */
  int32_t e_pitch;    /* (12,4): bytes per exponent-plane row, >= ceil(nb / 2);   */
                      /* (8,3): ignored                                           */
} seedlm_format;

/* Activation element types. */
enum { SEEDLM_F16 = 0, SEEDLM_BF16 = 1 };

/* Error codes. */
enum {
  SEEDLM_OK = 0,
  SEEDLM_EINVAL = -1,       /* null or misaligned pointer, bad size or field   */
  SEEDLM_EUNSUPPORTED = -2, /* format or size outside what the kernels handle  */
  SEEDLM_ECUDA = -3         /* a CUDA call failed; see seedlm_last_cuda_error  */
};

/* Prepares the current device (kernel attributes).  Idempotent; every entry
 * point calls it on first use of a device, so calling it is optional, but a
 * caller that captures CUDA graphs should call it once per device first. */
SEEDLM_API int seedlm_init(void);

/* W = decompressed weights, rows x cols, row-major with leading dimension ldw
 * (floats, >= cols).  Bit-exact.  (Eq (1) of the paperhub.cn thread, applied
 * to every block.) */
SEEDLM_API int seedlm_decompress(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                      float* W, int64_t ldw, seedlm_stream stream);

/* y = W x (batch 1).  x: cols elements of type x_dtype (SEEDLM_F16 or
 * SEEDLM_BF16); y: rows fp32.  The blocks are rebuilt on the fly and never
 * written out (paperhub.cn thread, authors' replies on inference and on the
 * custom decoding that avoids full-precision weights in memory).  Any width:
 * x is staged in shared memory as fp32 one column segment at a time.  Tall
 * 3-bit matrices (128 to 256 rows per SM) take a kernel that builds tables
 * of x's contribution per column block once per CTA and shares them across
 * its rows (same tolerance, a different fp32 summation order).  The
 * kernel is launched with programmatic dependent launch; it reads the
 * records and x only after waiting for the previous kernel in the stream,
 * so that kernel may write them (for example seedlm_encode, or a copy). */
SEEDLM_API int seedlm_gemv(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                const void* x, int x_dtype, float* y, seedlm_stream stream);

/* Several independent GEMVs in one launch (at most 8; all of one storage
 * format, the same C, P, K): y_k = W_k x_k for k < n.  fmts is a HOST array
 * of n formats; recs, eplanes (may be NULL for (8,3)), xs and ys are HOST
 * arrays of n DEVICE pointers, with the rules of seedlm_gemv for each entry
 * and one activation type for all.  One launch configuration serves the
 * whole batch (chosen from its largest product), so an entry's summation
 * order may differ from a separate seedlm_gemv call's: results agree with
 * separate calls within the products' tolerance, and bit for bit when the
 * entry alone would get the same configuration (as the large matrices of
 * one decoder layer do).  The kernel's setup (its decode tables in shared
 * memory) is paid once, and each CTA moves straight from its share of one
 * product to the next, with no launch or tail between them.  The pages name the extra
 * kernel launches of memory-bound work as a GPU cost of the method
 * (paperhub.cn review thread, authors' reply on GPU implementation
 * challenges); this is the library's answer for products that do not
 * depend on each other, e.g. the projections that share one input.  Empty
 * entries (rows == 0) are skipped; cols == 0 zeroes y_k. */
SEEDLM_API int seedlm_gemv_batch(int32_t n, const seedlm_format* fmts,
                                 const uint32_t* const* recs, const uint8_t* const* eplanes,
                                 const void* const* xs, int x_dtype, float* const* ys,
                                 seedlm_stream stream);

/* Y = X W^T for a small batch: X is M x cols (row-major, type x_dtype), Y is
 * M x rows fp32 (row-major), 1 <= M <= 64 -- the batched form of the
 * inference step of the paperhub.cn review thread (authors' reply on how
 * inference uses s and t: the blocks are rebuilt from seed and coefficients
 * and multiplied with the activations; a batch of M activation rows shares
 * every rebuilt block).  M = 1 runs the GEMV kernel; at 3 bits (C = 12,
 * P = 4) M = 2 to 4 run its extension on the CUDA cores (each rebuilt
 * weight pair feeds M packed fp32 FMAs; exact fp32 weights and
 * activations, the GEMV's accuracy; no workspace is used, so `workspace`
 * may then be NULL).  Otherwise the rebuilt weight tiles feed the tcgen05
 * tensor cores: kind::f16 MMAs on fp16 operands, W split exactly into two fp16 pieces of 2^6 W, fp32 accumulation
 * in TMEM.  fp16 X is used as it is; bf16 X is scaled per row by a power of
 * two that brings the row's largest finite magnitude to [2^15, 2^16) and
 * stored as fp16, exact for every element of at least 2^-32 times that
 * largest one (smaller elements round to fp16's subnormal grid, an error
 * below 2^-40 of the row's largest element); Y is scaled back exactly.  Two
 * launches: X is first written into the operand layout, then one CTA per SM
 * runs the GEMM.
 * `workspace` is device memory of at least
 * seedlm_gemm_smallM_workspace_bytes(fmt, M) bytes, 256-byte aligned.  It
 * holds per-tile counters, the rows' scale factors, X in the operand layout
 * and the partial tiles of row tiles shared by several CTAs: it must be
 * zero-filled before its first
 * use, every call leaves the counters at zero for the next, and calls sharing
 * one workspace must not run concurrently (calls on one stream never do). */
SEEDLM_API int seedlm_gemm_smallM(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                       const void* X, int x_dtype, int M, float* Y, void* workspace,
                       int64_t workspace_bytes, seedlm_stream stream);

/* Workspace bytes seedlm_gemm_smallM needs for this format and M on the
 * current device (HOST function; 0 for an empty matrix, for M = 1 (the GEMV)
 * and for M <= 4 at 3 bits (the CUDA-core kernel), negative on error). */
SEEDLM_API int64_t seedlm_gemm_smallM_workspace_bytes(const seedlm_format* fmt, int M);

/* Y = X W^T for any batch M >= 1 -- the same product as seedlm_gemm_smallM
 * (paperhub.cn review thread, authors' reply on how inference uses s and t),
 * extended to prefill-sized batches, where the rebuild of each weight tile is
 * shared by many rows of X.  X is M x cols (row-major, type x_dtype), Y is
 * M x rows fp32 (row-major).  M = 1, and M <= 4 at 3 bits, run as in
 * seedlm_gemm_smallM (the GEMV or its CUDA-core extension); otherwise the
 * rows of X go through the
 * tensor-core kernel of seedlm_gemm_smallM (same operand precision) in
 * passes of at most 256 rows, one after the other on the
 * stream: up to 64 rows per MMA as there, 65-128 rows as one N = 128 pass,
 * 129-256 as one N = 256 pass (units of 64 columns at 4 bits, 48 at 3 bits,
 * one accumulator in TMEM).  For M <= 64 the result is the one
 * seedlm_gemm_smallM gives.  `workspace`: device memory of at least
 * seedlm_gemm_workspace_bytes(fmt, M) bytes, 256-byte aligned, zero-filled
 * before its first use, with the sharing rules of seedlm_gemm_smallM. */
SEEDLM_API int seedlm_gemm(const seedlm_format* fmt, const uint32_t* rec, const uint8_t* eplane,
                           const void* X, int x_dtype, int M, float* Y, void* workspace,
                           int64_t workspace_bytes, seedlm_stream stream);

/* Workspace bytes seedlm_gemm needs for this format and M on the current
 * device (HOST function; 0 for an empty matrix, for M = 1 (the GEMV) and for
 * M <= 4 at 3 bits (the CUDA-core kernel), negative on error). */
SEEDLM_API int64_t seedlm_gemm_workspace_bytes(const seedlm_format* fmt, int M);

/* Same result as seedlm_gemm_smallM, for callers that cannot allocate device
 * memory -- e.g. code embedded in a host program that owns all of the GPU's
 * memory through its own pool, or a path where cudaMalloc's implicit device
 * synchronisation is not acceptable -- and so cannot provide a workspace.
 * It has no counterpart in the SeedLM pages; it only changes where the
 * workspace lives.  It is one array inside libseedlm.so (16 MiB + 64 KiB)
 * that every GPU which loads the library holds until the process exits; no
 * call allocates or frees anything.  Calls whose workspace would not fit
 * (seedlm_gemm_smallM_workspace_bytes(fmt, M) > 16 MiB + 64 KiB) return
 * SEEDLM_EUNSUPPORTED; use seedlm_gemm_smallM with a workspace for those.
 * Outside a stream capture every call looks up the array's device address
 * (cudaGetSymbolAddress); inside a capture the address from an earlier call
 * on the same device is used, so make one call on each device before
 * capturing it into a graph (a first call inside a capture returns
 * SEEDLM_EUNSUPPORTED).  Every call clears the counters and then reuses the same
 * array, so calls that overlap on the GPU (two streams, or unordered host
 * threads) race and give wrong results: order them, for example on one
 * stream. */
SEEDLM_API int seedlm_gemm_smallM_noalloc(const seedlm_format* fmt, const uint32_t* rec,
                                          const uint8_t* eplane, const void* X, int x_dtype,
                                          int M, float* Y, seedlm_stream stream);

/* The encoder: writes the records (and, for (12,4), the exponent plane) that
 * represent W (rows x cols fp32, row-major, leading dimension ldw >= cols,
 * device memory).  For every C-weight block w the seed s, coefficients q and
 * exponent e minimise ||w - U(s) q 2^-e||^2 over all 65,535 seeds and
 * e = 0..15, with q = clamp(round-half-even(pinv(U(s)) w 2^e), -8, 7); ties go
 * to the smallest seed, then the largest e (paperhub.cn thread, authors'
 * replies on parameter optimisation: a search over seeds, parallel over
 * blocks; the rounding and exponent rules are this library's reading).  A
 * tail block is fitted with its missing weights taken as zero.  rec/eplane
 * use the layout of seedlm_format; record slots past nb and exponent-plane
 * bytes past ceil(nb / 2) are left untouched.  err (optional, NULL or device
 * memory of rows x nb doubles, 8-byte aligned) receives each block's squared
 * error.  Each call allocates its seed tables (16 MiB for (8,3), 32 MiB for
 * (12,4)) on the stream with cudaMallocAsync and frees them the same way.
 * The search scores 65,535 seeds per block (a least-squares bound on the
 * tensor cores first, exact fp64 scoring for the seeds it cannot rule out),
 * so this is an offline (model-load) step, not part of the hot path. */
SEEDLM_API int seedlm_encode(const seedlm_format* fmt, const float* W, int64_t ldw, uint32_t* rec,
                             uint8_t* eplane, double* err, seedlm_stream stream);

/* Design-space search (the pages' discussion of seed bit-width K, block
 * size C and latent dimension P: paperhub.cn review thread, authors'
 * replies on compression time against those parameters; atlas.scime.ai
 * summary, "Limitations": the design was explored on Gaussian weights).
 * For each of nblocks blocks of C weights (W: nblocks x C fp32, row-major,
 * device memory) the search over all 2^K - 1 seeds of a K-bit register and
 * e = 0..15 returns the seed, the P coefficients q (int8, nblocks x P), the
 * exponent e and, if err != NULL (nblocks doubles, 8-byte aligned), the
 * squared error ||w - U(s) q 2^-e||^2, under the rounding and tie rules of
 * seedlm_encode.  The register shifts right and feeds the parity of its
 * tapped bits in at the top (taps: seedlm_lfsr_taps(K)); U(s)[c][p] =
 * (state_{pC+c} - 2^(K-1)) / 2^(K-1).  Supported: C in {8, 12, 16}, P in
 * {2, 3, 4}, 8 <= K <= 20 (else SEEDLM_EUNSUPPORTED).  The call allocates
 * its per-seed tables ((P*C + P*P) * (2^K - 1) doubles; 640 MiB at C = 16,
 * P = 4, K = 20) with cudaMallocAsync on the stream and frees them the same
 * way.  An offline tool (model-load or design time), not the hot path. */
SEEDLM_API int seedlm_search_blocks(int32_t C, int32_t P, int32_t K, const float* W,
                                    int64_t nblocks, uint32_t* seed, int8_t* q, uint8_t* e,
                                    double* err, seedlm_stream stream);

/* Tap mask of the K-bit register seedlm_search_blocks uses: 0x2D (bits 0, 2,
 * 3, 5, the workload's register) for K = 16; for other K, whose polynomial
 * the pages do not give, the smallest odd mask whose register visits all
 * 2^K - 1 nonzero states.  0 for K outside 8..20.  HOST function. */
SEEDLM_API uint32_t seedlm_lfsr_taps(int32_t K);

/* Failure-path self test (no counterpart in the pages): launches one small
 * kernel whose bounded mbarrier wait -- the wait the tensor-core GEMM uses,
 * with its TMEM allocation -- waits for an arrival that never comes and gives
 * up after limit_ns nanoseconds (1e3 .. 1e8, else SEEDLM_EINVAL).  Afterwards
 * seedlm_device_error reports 1 and the context stays usable: this is how a
 * stuck hand-over surfaces to the caller, without a trap or a hang. */
SEEDLM_API int seedlm_selftest_wait_timeout(int64_t limit_ns, seedlm_stream stream);

/* Reads and clears the device-side error flags of the current device into
 * *flag: bit 0 (value 1) if a kernel gave up waiting on one of its own
 * barriers, bit 1 (value 2) if a kernel of a checked build (below) computed a
 * memory index outside the buffers its arguments describe, or a
 * shared-memory index outside its launch's allocation, and skipped that
 * access.  The outputs of such a call are undefined.  0 if neither happened.
 * HOST function; synchronous. */
SEEDLM_API int seedlm_device_error(int* flag);

/* Failure-path self test of the checked build: one kernel thread compares
 * index with extent exactly as the kernels' bounds checks do, with no memory
 * access behind it.  In a checked build, index >= extent then makes
 * seedlm_device_error report bit 1; other builds compile the check away and
 * report nothing.  Negative arguments return SEEDLM_EINVAL. */
SEEDLM_API int seedlm_selftest_bounds_check(int64_t index, int64_t extent, seedlm_stream stream);

/* 1 if this library was compiled with -DSEEDLM_CHECK=1: every kernel then
 * compares each global and shared memory index it computes with the extent
 * of the buffer before the access (slower; for testing), else 0. */
SEEDLM_API int seedlm_checked_build(void);

/* Reference point, not part of the method: y = W x with W dense fp16
 * (rows x cols, row-major, leading dimension ldw halves, 16-byte aligned with
 * ldw % 8 == 0), x fp16 (cols), y fp32 (rows). */
SEEDLM_API int seedlm_dense_gemv_f16(int32_t rows, int32_t cols, const uint16_t* W, int64_t ldw,
                          const uint16_t* x, float* y, seedlm_stream stream);

/* Bytes of compressed storage one row needs at the ideal packing
 * ((K + 4P + 4) * nb / 8, no pitch padding) and as laid out (4 * rec_pitch +
 * e_pitch).  HOST function; returns -1 on a bad format. */
SEEDLM_API int64_t seedlm_row_bytes_ideal(const seedlm_format* fmt);
SEEDLM_API int64_t seedlm_row_bytes_stored(const seedlm_format* fmt);

/* Static description of an error code (never NULL). */
SEEDLM_API const char* seedlm_strerror(int code);

/* The cudaError_t of the last SEEDLM_ECUDA on this host thread (0 if none). */
SEEDLM_API int seedlm_last_cuda_error(void);

/* Number of kernel launches this library has enqueued since load (all
 * threads); used to count the library's launches in a timed region. */
SEEDLM_API int64_t seedlm_launch_count(void);

/* Releases nothing that outlives the process today; kept for symmetry with
 * seedlm_init.  Safe to call more than once. */
SEEDLM_API void seedlm_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* SEEDLM_H */
