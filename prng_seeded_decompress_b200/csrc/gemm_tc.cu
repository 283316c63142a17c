// gemm_tc.cu -- Y = X W^T for a small batch on the 5th-generation tensor
// cores (tcgen05), with W rebuilt on the fly.
//
// Where the batch makes the product a real contraction (several rows of X
// share every rebuilt weight), the reconstructed tiles feed tcgen05.mma
// (paperhub.cn review thread: the weights are rebuilt from s and t and then
// used to compute the activations).  The MMAs are kind::f16 (K = 16) on
// fp16 operands:
//
//   * W: 2^6 W = p1 + p2, two fp16 pieces (11 significant bits each; a
//     rebuilt weight has at most 20, and the 2^6 keeps the smallest weight
//     quantum, 2^-30, at or above fp16's 2^-24).  Every product of a piece
//     and an activation is exact in the fp32 accumulator.
//   * X: fp16 activations as they are; bf16 activations scaled per row n by
//     a power of two 2^s_n that brings the row's largest finite magnitude to
//     [2^15, 2^16) and stored as fp16.  A bf16 value has 8 significant bits,
//     so every element of at least 2^-32 times its row's largest is exact;
//     smaller ones round to fp16's subnormal grid, an error below 2^-40 of
//     the row's largest element.
//   * Y = acc * 2^-(6 + s_n), applied as two exact power-of-two products.
//
// Two pieces instead of three bf16 pieces cut the MMAs per K step from 3 to
// 2 and the producers' split from ten instructions per weight pair to six.
//
// One call is two launches:
//
//   1. stage_x_kernel writes X (M x cols) into the workspace in the
//      tensor-core operand layout, one contiguous fp16 slab per K chunk (NB x
//      KC elements, NB = M rounded up to 16, zero-padded), and the two scale
//      factors of each row.  A CTA covers one row n and a range of its
//      columns; for bf16 X it first takes the maximum over the whole row.
//   2. gemm_tc_kernel, one CTA per SM.  The work is the list of
//      (128-row tile, K chunk) units in tile-major order, cut into equal
//      contiguous ranges, one per CTA ("stream-K"), so every SM gets the same
//      number of units whatever the shape.  Inside a CTA:
//        * 16 producer warps rebuild the unit's 128 x KC weights exactly in
//          fp32 (seedlm_device.cuh) with the lane-replicated decode tables
//          (rep_tables.cuh: one conflict-free shared-memory wavefront per
//          lookup), split them into the two fp16 pieces, pack two K
//          neighbours per 32-bit word and store them straight into tensor
//          memory with tcgen05.st (for C = 8 one asm statement per two
//          blocks: hi = the weight truncated to fp16, lo from a
//          mixed-precision FMA, both written into the store's source
//          registers) -- A operand stages, 128 lanes = rows.  Warp w owns TMEM lanes 32(w%4).. and a quarter
//          (w/4) of the chunk's blocks.  The producers set the pace: measured
//          about 1,350 cycles of rebuild per warp and unit plus 250 waiting
//          for the slowest warp of the stage, at about 60 % issue use.
//        * one warp issues the MMAs (M = 128, N = NB, A from TMEM, B = X
//          slab from shared memory), both pieces into the same fp32
//          accumulator in TMEM, a unit's MMAs in one asm statement with one
//          elect.  An MMA of this shape keeps the tensor core busy ~32
//          cycles whatever N (<= 64) and K, so the MMA count, not M*N*K, sets
//          the tensor-core time; issuing a unit's 16 takes ~900 cycles of the
//          warp that shares its scheduler with four producer warps.
//        * one thread keeps the X slabs coming, a few chunks ahead, with bulk
//          copies.
//        * stages are handed over with mbarriers only (A stage full: all 16
//          producer warps arrived; A stage / X slab free: tcgen05.commit of the
//          MMAs that read it), so no warp waits for the whole CTA.
//        * the accumulator is double-buffered in TMEM.  At the end of each
//          tile segment the MMA warp commits to an "accumulator full"
//          barrier, and four epilogue warps of their own read it out and
//          scale it while the producers go on with the next segment: a tile
//          owned by one CTA goes straight to Y; otherwise each CTA writes a
//          partial tile to the workspace and the last of the tile's CTAs to
//          arrive (atomic counter) adds the partials in CTA order -- a fixed
//          order, so every call gives the same bits -- writes Y and resets
//          the counter.
//   Every mbarrier wait is bounded; a wait that gives up raises the library's
//   device error flag, and TMEM is always released.
//
//   The GEMM is launched with programmatic stream serialization: its
//   prologue (tables, barriers, TMEM) and the producers' first units overlap
//   stage_x_kernel.  The producers read only the records, which the kernel
//   before stage_x_kernel (a plain launch, so fully finished) may have
//   written; the X slabs and scale factors are read after griddepcontrol.wait.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "rep_tables.cuh"
#include "seedlm_device.cuh"
#include "seedlm_internal.h"
#include "tcgen05.cuh"

namespace seedlm {

__device__ unsigned int g_tc_error = 0;

SEEDLM_CHECK_FLAG(gemm_tc)

namespace {

constexpr int kTileM = 128;
// Warp roles: producer warps (a multiple of 4: each TMEM lane quarter gets
// the same number), then the MMA warp, the X loader warp and four epilogue
// warps.  (24 producer warps on 96-column C = 8 units, 64 registers each,
// measured 13 % slower than 16 on 128-column units.)
template <int C>
struct Roles {
  static constexpr int kProd = 16;
  static constexpr int kMma = kProd;         // issues the MMAs (one thread)
  static constexpr int kLoader = kProd + 1;  // copies the X slabs (one thread)
  static constexpr int kEpi0 = kProd + 2;    // four warps drain the accumulators
  static constexpr int kThreads = (kProd + 6) * 32;
  static_assert(kProd % 4 == 0, "whole lane quarters");
};
constexpr int kTmemCols = 512;
constexpr int kMaxNB = 256;      // batch rows of one pass (the MMA's largest N)
constexpr int kShift = 6;        // the pieces are of 2^kShift W
constexpr int kMaxXS = 5;        // X slabs in shared memory, at most
constexpr int kHdrBytes = 2304;  // mbarriers, TMEM slot, row scales, at the allocation's start
constexpr uint32_t kSmemLimit = rep::kSmemBase + 232448;  // end of the largest allocation (B200)
constexpr int kRecAhead = 3;   // units of records a producer thread has in flight (2: 1-2 % slower)
constexpr uint64_t kWaitLimit = 2000000000ull;  // ns an mbarrier wait may take before giving up

// Batch rows NB (a pass's M rounded up: 16, 32, 48, 64, 128 or 256) ->
// K columns per unit and blocks per producer thread and unit.  Up to 128
// rows: units of 128 (C = 8) or 96 (C = 12) columns.  Above: half-width
// units, so that two X slabs of 32 KB still fit beside the decode tables.
template <int C, int NB>
struct TcCfg {
  static constexpr int BPT = (NB > 128) ? (C == 8 ? 2 : 1) : (C == 8 ? 4 : 2);
  static constexpr int KC = 4 * BPT * C;  // 128, 64 (C = 8); 96, 48 (C = 12)
};

struct TcGeom {
  int rows, cols, nb, rec_pitch, e_pitch, M;
  int nchunks, tiles;
  long long units;  // tiles * nchunks
  int segs_max;     // most tiles any one CTA touches
};

// Shared memory, by absolute shared address (the dynamic allocation starts
// at rep::kSmemBase; checked at entry):
//   [kSmemBase, +kHdrBytes)           mbarriers, TMEM base, flags, row scales
//   [kSmemBase + kHdrBytes, tables)   X slabs, as many as fit
//   [tables, rep::kEnd)               lane-replicated decode tables
//   [rep::kEnd, ...)                  the remaining X slabs
// TMEM: AS A stages of two pieces (KC/2 columns each: two fp16 per 32-bit
// column), then NACC accumulators of ACC fp32 columns (two, so that one
// segment's epilogue overlaps the next segment, when they fit).
template <int C, int NB>
struct TcSmem {
  static constexpr int KC = TcCfg<C, NB>::KC;
  static constexpr int BPT = TcCfg<C, NB>::BPT;
  static constexpr int SBO = KC * 16;      // bytes between 8-row groups of X (KC/8 core matrices)
  static constexpr int XB = NB * KC * 2;   // one X slab (fp16)
  static constexpr int PIECE_COLS = KC / 2;
  static constexpr int STAGE_COLS = 2 * PIECE_COLS;
  static constexpr int ACC = NB < 64 ? 64 : NB;
  static constexpr int NACC = (2 * ACC + 2 * STAGE_COLS <= kTmemCols) ? 2 : 1;
  static constexpr int AS = (kTmemCols - NACC * ACC) / STAGE_COLS;
  static constexpr int D_COL = AS * STAGE_COLS;  // first accumulator column
  static constexpr uint32_t SLAB_A = rep::kSmemBase + kHdrBytes;
  static constexpr uint32_t TAB = rep::tables_begin<C>();
  static constexpr int A_CAP = (int)((TAB - SLAB_A) / XB);          // slabs below the tables
  static constexpr int B_CAP = (int)((kSmemLimit - rep::kEnd) / XB);  // slabs above them
  static constexpr int XS = A_CAP + B_CAP < kMaxXS ? A_CAP + B_CAP : kMaxXS;
  static constexpr int SLABS_A = A_CAP < XS ? A_CAP : XS;
  // mbarriers: xfull[XS] xfree[XS] afull[AS] afree[AS] dfree[NACC] dfull[NACC]
  static constexpr int NBAR = 2 * XS + 2 * AS + 2 * NACC;
  static constexpr uint32_t BAR = rep::kSmemBase;
  static constexpr uint32_t SLOT = BAR + 8 * NBAR;  // TMEM base, last-CTA flag, give-up flag
  static constexpr uint32_t YSCALE = rep::kSmemBase + 256;  // NB float2: the rows' output scales
  static constexpr uint32_t END = XS > SLABS_A ? rep::kEnd + (uint32_t)(XS - SLABS_A) * XB : rep::kEnd;
  static constexpr int TOTAL = (int)(END - rep::kSmemBase);
  __host__ __device__ static constexpr uint32_t slab(int s) {
    return s < SLABS_A ? SLAB_A + (uint32_t)s * XB : rep::kEnd + (uint32_t)(s - SLABS_A) * XB;
  }
  static_assert(XS >= 2, "X slabs are double-buffered at least");
  static_assert(AS >= 2, "A stages are double-buffered at least");
  static_assert(SLOT + 16 <= YSCALE && YSCALE + 8 * kMaxNB <= SLAB_A, "header");
  static_assert(D_COL + NACC * ACC <= kTmemCols, "TMEM budget");
  static_assert(NB <= kMaxNB && NB <= ACC, "one accumulator holds the pass");
  static_assert(KC == Roles<C>::kProd / 4 * BPT * C, "each producer warp of a lane quarter takes BPT blocks");
  static_assert(KC % 16 == 0, "whole K = 16 MMA steps");
  static_assert(SLAB_A % 16 == 0 && XB % 16 == 0, "bulk copies and descriptors need 16-byte alignment");
};

// Byte offset of X element (n, k) inside a slab (K-major core matrices:
// 8 rows x 16 bytes = 8 elements, adjacent along K at 128 B, 8-row groups at
// SBO = KC * 16 bytes).
template <int KC>
__host__ __device__ constexpr int slab_byte(int n, int k) {
  return (n >> 3) * (KC * 16) + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

// 2^k as a float, -126 <= k <= 127.
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float((uint32_t)(127 + k) << 23); }

// Largest finite magnitude (as bf16 bits without the sign) among two packed
// bf16 values; inf and NaN count as 0.
__device__ __forceinline__ uint32_t finite_mag2(uint32_t v) {
  const uint32_t a = v & 0x7FFFu, b = (v >> 16) & 0x7FFFu;
  return max(a < 0x7F80u ? a : 0u, b < 0x7F80u ? b : 0u);
}

// One CTA per (row n of the padded batch, column part).  Writes the row's
// fp16 slab entries for its part (zeros past M rows and past cols) and, part
// 0, the row's output scale factors (f1, f2): Y = (acc * f1) * f2.  bf16 X
// needs the row's largest magnitude: every CTA reads the whole row for it,
// or, when the row's parts form a thread-block cluster (`clustered`), each
// CTA takes the maximum over its own part and reads the others' from their
// shared memory, so the row is read once (without: 51 MB and ~10 us for 64
// rows of 28672 columns in 14 parts).
template <int KC, int NB>
__global__ void __launch_bounds__(256)
stage_x_kernel(const uint16_t* __restrict__ X, int M, int cols, int nchunks, int is_bf16,
               int clustered, int parts, int vec, unsigned char* __restrict__ Xs,
               float2* __restrict__ yscale) {
  // The GEMM may start its prologue at once; it reads Xs and yscale only after
  // griddepcontrol.wait, i.e. after this grid has finished.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ uint32_t red[8];
  __shared__ uint32_t part_max;
  const int n = blockIdx.x / parts, part = blockIdx.x - n * parts;
  const uint16_t* row = X + (size_t)n * cols;
  const int groups = nchunks * (KC / 8);  // 8-column groups of the padded row
  const int g0 = (int)((long long)part * groups / parts);
  const int g1e = (int)((long long)(part + 1) * groups / parts);
  int s = 0;  // x is stored as x * 2^s
  if (is_bf16) {
    namespace cg = cooperative_groups;
    // The maximum over this CTA's own part when the row's parts form a
    // cluster, else over the whole row.
    uint32_t m = 0;
    if (n < M && clustered) {
      for (int gi = g0 + threadIdx.x; gi < g1e; gi += blockDim.x) {
        const int col = 8 * gi;
        if (vec && col + 8 <= cols) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + col));
          m = max(m, max(max(finite_mag2(v.x), finite_mag2(v.y)), max(finite_mag2(v.z), finite_mag2(v.w))));
        } else {
          for (int u = 0; u < 8 && col + u < cols; ++u) m = max(m, finite_mag2(row[col + u]));
        }
      }
    } else if (n < M && vec) {
      const uint4* r4 = reinterpret_cast<const uint4*>(row);
      for (int i = threadIdx.x; i < cols / 8; i += blockDim.x) {
        const uint4 v = __ldg(r4 + i);
        m = max(m, max(max(finite_mag2(v.x), finite_mag2(v.y)), max(finite_mag2(v.z), finite_mag2(v.w))));
      }
    } else if (n < M) {
      for (int k = threadIdx.x; k < cols; k += blockDim.x) m = max(m, finite_mag2(row[k]));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = max(m, red[w]);
    if (clustered) {
      const cg::cluster_group cluster = cg::this_cluster();
      if (threadIdx.x == 0) part_max = m;
      cluster.sync();  // every part's maximum is in its CTA's shared memory
      for (int r = 0; r < parts; ++r) m = max(m, *cluster.map_shared_rank(&part_max, r));
    }
    if (m) {
      const int E = max((int)(m >> 7), 1) - 127;  // the largest has its leading bit at or below 2^E
      s = 15 - E;                                 // -112 <= s <= 141
    }
  }
  const int s1 = s / 2, s2 = s - s1;
  if (part == 0 && threadIdx.x == 0)
    yscale[n] = make_float2(exp2i(-(kShift + s1)), exp2i(-s2));
  const float g1 = exp2i(s1), g2 = exp2i(s2);
  for (int gi = g0 + threadIdx.x; gi < g1e; gi += blockDim.x) {
    const int col = 8 * gi;
    uint16_t h[8];
    if (n < M && vec && col + 8 <= cols) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + col));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 8; ++u) h[u] = (uint16_t)(w[u >> 1] >> (16 * (u & 1)));
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) h[u] = (n < M && col + u < cols) ? row[col + u] : (uint16_t)0;
    }
    uint32_t o[4];
#pragma unroll
    for (int u = 0; u < 8; u += 2) {
      uint32_t a = h[u], b = h[u + 1];
      if (is_bf16) {
        const __half2 c = __floats2half2_rn(__uint_as_float(a << 16) * g1 * g2,
                                            __uint_as_float(b << 16) * g1 * g2);
        o[u >> 1] = *reinterpret_cast<const uint32_t*>(&c);
      } else {
        o[u >> 1] = a | (b << 16);
      }
    }
    const int chunk = col / KC;
    const size_t xb = (size_t)chunk * (NB * KC * 2) + slab_byte<KC>(n, col - chunk * KC);
    if (SEEDLM_IN_BOUNDS(g_check_flag, xb + 15, (size_t)nchunks * (NB * KC * 2)))
      *reinterpret_cast<uint4*>(Xs + xb) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  // No CTA of the cluster leaves while another may still read its maximum.
  if (is_bf16 && clustered) cooperative_groups::this_cluster().sync();
}

__device__ __forceinline__ long long unit_begin(int cta, long long units, int ctas) {
  return (long long)cta * units / ctas;
}
// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long u, long long units, int ctas) {
  return (int)(((u + 1) * ctas + units - 1) / units) - 1;
}

// The two pieces of two rebuilt weights (K neighbours) given as
// magic-biased bit patterns t (weight * 2^6 = t + nm): the top 11
// significant bits h, then the rest l (at most 9 bits).  Both are exact in
// fp16 and h + l is exact.  neg1 holds (-1, -1).
__device__ __forceinline__ void f32_pieces(int32_t t0, int32_t t1, float2 nm, float2 neg1, float& h0,
                                           float& h1, float& l0, float& l1) {
  const float2 w = __fadd2_rn(make_float2(__int_as_float(t0), __int_as_float(t1)), nm);
  h0 = __uint_as_float(__float_as_uint(w.x) & 0xFFFFE000u);
  h1 = __uint_as_float(__float_as_uint(w.y) & 0xFFFFE000u);
  const float2 l = __ffma2_rn(make_float2(h0, h1), neg1, w);
  l0 = l.x;
  l1 = l.y;
}

// The same pieces converted to fp16 and packed two per 32-bit word, the
// lower K index in the low half.
__device__ __forceinline__ void fp16_pieces(int32_t t0, int32_t t1, float2 nm, float2 neg1,
                                            uint32_t& hi, uint32_t& lo) {
  float h0, h1, l0, l1;
  f32_pieces(t0, t1, nm, neg1, h0, h1, l0, l1);
  const __half2 ph = __floats2half2_rn(h0, h1);
  const __half2 pl = __floats2half2_rn(l0, l1);
  hi = *reinterpret_cast<const uint32_t*>(&ph);
  lo = *reinterpret_cast<const uint32_t*>(&pl);
}

// Weights c and c + 1 of a C = 8 block as 2^6 W in fp32 (exact), into w[c], w[c + 1].
template <int c>
__device__ __forceinline__ void w64_pair(const BlockC8& blk, float2 nm, float* w) {
  const float2 t = __fadd2_rn(
      make_float2(__int_as_float(weight_bits_c8<c>(blk)), __int_as_float(weight_bits_c8<c + 1>(blk))), nm);
  w[c] = t.x;
  w[c + 1] = t.y;
}

// (tile, chunk) of consecutive units, advanced without dividing: a 64-bit
// division costs hundreds of instructions, more than rebuilding a unit.
struct UnitCursor {
  int tile, chunk;
  __device__ __forceinline__ void next(int nchunks) {
    if (++chunk == nchunks) {
      chunk = 0;
      ++tile;
    }
  }
};

template <int C>
struct RecUnit {
  uint32_t r[C == 8 ? 4 : 2];  // the thread's records of this unit
  uint32_t e;                  // C = 12: their exponent byte
};

template <int C, int NB>
__global__ void __launch_bounds__(Roles<C>::kThreads, 1)
gemm_tc_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
               const unsigned char* __restrict__ Xs, const float2* __restrict__ yscale,
               float* __restrict__ Y, float* __restrict__ partial,
               unsigned int* __restrict__ counters, TcGeom g) {
  using L = TcSmem<C, NB>;
  using R = Roles<C>;
  constexpr int KC = L::KC, AS = L::AS, BPT = L::BPT, XS = L::XS, NACC = L::NACC, ACC = L::ACC;
  constexpr int kThreads = R::kThreads, kProdWarps = R::kProd, kMmaWarp = R::kMma,
                kLoaderWarp = R::kLoader, kEpiWarp0 = R::kEpi0;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ctas = gridDim.x;
  // The shared-memory map is by absolute address: the allocation must start
  // at rep::kSmemBase and hold the whole map (checked before any barrier or
  // TMEM exists, so leaving is safe).
  if (tc::smem_u32(smem) != rep::kSmemBase) {
    if (tid == 0) atomicOr(&g_tc_error, 1u);
    return;
  }
  if (!SEEDLM_IN_BOUNDS(g_check_flag, L::TOTAL - 1, seedlm_dynamic_smem_bytes())) return;
  const long long u_begin = unit_begin(blockIdx.x, g.units, ctas);
  const int n_units = (int)(unit_begin(blockIdx.x + 1, g.units, ctas) - u_begin);
  const int t_first = (int)(u_begin / g.nchunks);
  const UnitCursor c0{t_first, (int)(u_begin - (long long)t_first * g.nchunks)};

  // Producer warps: their first records are requested before the prologue
  // (tables, barriers, TMEM), which then hides the memory latency.  The
  // records are read before griddepcontrol.wait: the kernel before
  // stage_x_kernel, a plain launch, has finished writing them.
  const int lq = warp & 3, kq = warp >> 2;
  const int prow = 32 * lq + lane;  // TMEM lane = row in the tile
  const uint32_t lane4 = (uint32_t)lane << 2, lane8 = (uint32_t)(lane & 15) << 3;
  const float2 neg1 = make_float2(-1.f, -1.f);
  auto load_rec = [&](const UnitCursor& u, RecUnit<C>& p) {
    const int gr = u.tile * kTileM + prow;
    const int b0 = u.chunk * (KC / C) + kq * BPT;  // a multiple of BPT
    // The thread's last record and its exponent byte lie inside row gr.
    const bool ok_ = gr < g.rows && b0 < g.nb &&
                     SEEDLM_IN_BOUNDS(g_check_flag, b0 + BPT - 1, g.rec_pitch) &&
                     (C == 8 || SEEDLM_IN_BOUNDS(g_check_flag, b0 >> 1, g.e_pitch));
    const uint32_t* src = rec + (size_t)gr * g.rec_pitch + b0;
    // b0 is a multiple of BPT, so each load is aligned to its width.
    if constexpr (C == 8 && BPT == 4) {
      const uint4 v = ok_ ? ld_stream_u4(src) : make_uint4(0u, 0u, 0u, 0u);
      p.r[0] = v.x; p.r[1] = v.y; p.r[2] = v.z; p.r[3] = v.w;
      p.e = 0;
    } else if constexpr (C == 8) {
      static_assert(BPT == 2, "C = 8 takes two or four blocks per thread");
      const uint2 v = ok_ ? ld_stream_u2(src) : make_uint2(0u, 0u);
      p.r[0] = v.x; p.r[1] = v.y;
      p.e = 0;
    } else if constexpr (BPT == 2) {
      // b0 is even: one 8-byte load; the exponent byte holds block b0 in
      // its low nibble and b0 + 1 in its high nibble.
      const uint2 v = ok_ ? ld_stream_u2(src) : make_uint2(0u, 0u);
      p.r[0] = v.x; p.r[1] = v.y;
      p.e = ok_ ? (uint32_t)ld_stream_u8(eplane + (size_t)gr * g.e_pitch + (b0 >> 1)) : 0u;
    } else {
      // One block: a 4-byte load, the exponent from the nibble of b0's parity.
      static_assert(BPT == 1, "C = 12 takes one or two blocks per thread");
      p.r[0] = ok_ ? ld_stream_u1(src) : 0u;
      const uint32_t eb = ok_ ? (uint32_t)ld_stream_u8(eplane + (size_t)gr * g.e_pitch + (b0 >> 1)) : 0u;
      p.e = eb >> (4 * (b0 & 1));
    }
  };

  RecUnit<C> ring[kRecAhead];
  UnitCursor rc = c0;  // next unit whose records are loaded
  if (warp < kProdWarps) {
#pragma unroll
    for (int k = 0; k < kRecAhead; ++k)
      if (k < n_units) {
        load_rec(rc, ring[k]);
        rc.next(g.nchunks);
      }
  }

  rep::fill_rep_tables<C, kShift>(smem, tid, kThreads);
  const uint32_t bar = L::BAR;
  // xfull: X slab landed.  xfree: the MMAs that read the slab completed.
  // afull: all producer warps stored the A stage.  afree: the unit's MMAs
  // completed: its A stage may be reused.  dfull: a segment's MMAs completed,
  // its accumulator is final.  dfree: the epilogue warps have read it out.
  auto xfull = [&](int s) { return bar + 8 * s; };
  auto xfree = [&](int s) { return bar + 8 * (XS + s); };
  auto afull = [&](int s) { return bar + 8 * (2 * XS + s); };
  auto afree = [&](int s) { return bar + 8 * (2 * XS + AS + s); };
  auto dfree = [&](int b) { return bar + 8 * (2 * XS + 2 * AS + b); };
  auto dfull = [&](int b) { return bar + 8 * (2 * XS + 2 * AS + NACC + b); };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + (L::SLOT - rep::kSmemBase));
  if (tid == 0) {
    for (int s = 0; s < XS; ++s) {
      tc::mbar_init(xfull(s), 1);
      tc::mbar_init(xfree(s), 1);
    }
    for (int s = 0; s < AS; ++s) {
      tc::mbar_init(afull(s), kProdWarps);
      tc::mbar_init(afree(s), 1);
    }
    for (int b = 0; b < NACC; ++b) {
      tc::mbar_init(dfree(b), 4);
      tc::mbar_init(dfull(b), 1);
    }
    tc::fence_mbar_init();
    slot[2] = 0u;  // give-up flag shared by all bounded waits
  }
  if (warp == 0) tc::tmem_alloc(L::SLOT, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = slot[0];
  volatile uint32_t* abort_flag = slot + 2;
  bool ok = true;

  if (warp == kLoaderWarp) {
    // ------------------------------------------------ X slabs
    if (lane == 0) {
      UnitCursor xc = c0;
      // Xs is written by the previous kernel on the stream.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int j = 0; j < n_units; ++j, xc.next(g.nchunks)) {
        const int s = j % XS;
        if (j >= XS)  // the slab's previous unit (j - XS) has finished its MMAs
          ok = tc::mbar_wait_or_abort(xfree(s), ((j / XS) - 1) & 1, kWaitLimit, abort_flag) && ok;
        if (SEEDLM_IN_BOUNDS(g_check_flag, xc.chunk, g.nchunks)) {
          tc::mbar_arrive_expect_tx(xfull(s), L::XB);
          tc::bulk_g2s(L::slab(s), Xs + (size_t)xc.chunk * L::XB, L::XB, xfull(s));
        } else {
          tc::mbar_arrive(xfull(s));  // checked build: no copy, the hand-over still completes
        }
      }
      // Every copy this thread issued has landed before the CTA may exit
      // (bounded, and not cut short by the give-up flag).
      for (int s = 0; s < XS && s < n_units; ++s) {
        const int k = (n_units - 1 - s) / XS;  // last load into slab s
        ok = tc::mbar_wait(xfull(s), k & 1, kWaitLimit) && ok;
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issue
    // The whole warp runs this loop with warp-uniform values (so they can
    // stay in uniform registers); one elected lane issues each MMA/commit.
    {
      constexpr uint32_t idesc = tc::idesc_f16(NB, 0);
      int seg = 0;
      UnitCursor mc = c0;
      for (int i = 0; i < n_units; ++i, mc.next(g.nchunks)) {
        const bool first = i == 0 || mc.chunk == 0;
        if (first && i > 0) ++seg;
        const int db = seg % NACC;
        if (first && seg >= NACC)  // accumulator db was last used by segment seg - NACC
          ok = tc::mbar_wait_or_abort(dfree(db), ((seg / NACC) - 1) & 1, kWaitLimit, abort_flag) && ok;
        const int xs = i % XS, as = i % AS;
        if (!tc::mbar_try_wait2(xfull(xs), (i / XS) & 1, afull(as), (i / AS) & 1)) {
          ok = tc::mbar_wait_or_abort(xfull(xs), (i / XS) & 1, kWaitLimit, abort_flag) && ok;
          ok = tc::mbar_wait_or_abort(afull(as), (i / AS) & 1, kWaitLimit, abort_flag) && ok;
        }
        __syncwarp();  // reconverge before the elected issue
        tc::fence_after_sync();
        // The issue rate bounds the tensor core here, so everything but the
        // MMAs is computed up front.
        const uint32_t a0 = tmem + as * L::STAGE_COLS;
        const uint32_t d = tmem + L::D_COL + ACC * db;
        const uint64_t bd = tc::smem_desc(L::slab(xs), 128, L::SBO);
        const uint32_t acc0 = first ? 0u : 1u;
        // The unit's MMAs in one statement with one elect (measured: the
        // per-MMA form costs the issuing warp 45 % more cycles).
        static_assert(L::PIECE_COLS == KC / 2, "the helpers' piece stride");
        if constexpr (KC == 128)
          tc::mma_f16_ts_warp_8x2(d, a0, bd, idesc, acc0);
        else if constexpr (KC == 96)
          tc::mma_f16_ts_warp_6x2(d, a0, bd, idesc, acc0);
        else if constexpr (KC == 64)
          tc::mma_f16_ts_warp_4x2(d, a0, bd, idesc, acc0);
        else
          tc::mma_f16_ts_warp_3x2(d, a0, bd, idesc, acc0);
        static_assert(KC == 128 || KC == 96 || KC == 64 || KC == 48, "a unit's MMA count");
        tc::mma_commit_warp(afree(as));  // A stage free
        tc::mma_commit_warp(xfree(xs));  // X slab free
        if (i == n_units - 1 || mc.chunk == g.nchunks - 1)
          tc::mma_commit_warp(dfull(db));  // the segment's accumulator is final
      }
      // The CTA releases TMEM only after its last MMAs have completed
      // (bounded, not cut short by the give-up flag).
      if (n_units > 0) {
        const int last = n_units - 1;
        ok = tc::mbar_wait(afree(last % AS), (last / AS) & 1, kWaitLimit) && ok;
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ epilogue
    // Warp kEpiWarp0 + j reads TMEM lanes 32 (warp % 4).. (a warp reaches
    // the lane quarter of its warp index modulo 4), so the four warps cover
    // all 128 rows of the tile.  Each segment's accumulator is read out 16
    // columns at a time, scaled by the rows' factors and written.
    const int eq = warp & 3;
    const int row = 32 * eq + lane;
    const bool leader = warp == kEpiWarp0 && lane == 0;
    // The rows' scale factors, written by the previous kernel on the stream,
    // into shared memory once.
    float2* ys = reinterpret_cast<float2*>(smem + (L::YSCALE - rep::kSmemBase));
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = tid - kEpiWarp0 * 32; i < NB; i += 128) ys[i] = __ldcg(yscale + i);
    tc::named_sync(128);
    // Measured: the fast fixup below pays at N = 16, 32 and 256; at 48 to 128
    // its code costs the producers registers (spills) and the kernel time.
    constexpr bool kFastFixup = NB <= 32 || NB == 256;
    auto epilogue = [&](int seg, int tile, bool final_seg) {
      const int db = seg % NACC;
      const int gr = tile * kTileM + row;
      const int first = unit_owner((long long)tile * g.nchunks, g.units, ctas);
      const int last = unit_owner((long long)(tile + 1) * g.nchunks - 1, g.units, ctas);
      float* mine = partial + ((size_t)blockIdx.x * g.segs_max + seg) * (NB * kTileM);
      // Extents: Y holds M x rows floats; the partial tiles ctas x segs_max
      // tiles of NB x 128 floats (one per segment of each CTA).
      SEEDLM_CHECK_ONLY(const size_t y_n = (size_t)g.M * g.rows;
                        const size_t part_n = (size_t)ctas * g.segs_max * (NB * kTileM);
                        const size_t mine_off = ((size_t)blockIdx.x * g.segs_max + seg) * (NB * kTileM);)
      // The CTA's last segment, when it starts the tile and other CTAs finish
      // it: they began with it, so they have usually counted their partials
      // long before.  If all of them have, this CTA adds the partials straight
      // away, its own first and from TMEM (no later segment reuses the
      // accumulator), and neither writes its own partial nor waits for that
      // write.  Same sum, in the same CTA order, as the general path below.
      if (kFastFixup && final_seg && first != last && first == (int)blockIdx.x) {
        if (leader) {
          const bool all_in = SEEDLM_IN_BOUNDS(g_check_flag, tile, g.tiles) &&
                              atomicAdd(&counters[tile], 0u) == (unsigned)(last - first);
          if (all_in) __threadfence();
          slot[1] = all_in ? 1u : 0u;
        }
        tc::named_sync(128);
        const bool all_in = slot[1] != 0u;
        tc::named_sync(128);  // slot[1] is rewritten below
        if (all_in) {
          ok = tc::mbar_wait_or_abort(dfull(db), (seg / NACC) & 1, kWaitLimit, abort_flag) && ok;
          tc::fence_after_sync();
#pragma unroll 1
          for (int n16 = 0; n16 < NB / 16; ++n16) {
            float v[16];
            tc::tmem_ld16(tmem + ((uint32_t)(32 * eq) << 16) + L::D_COL + ACC * db + 16 * n16, v);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float2 f = ys[16 * n16 + q];
              v[q] = v[q] * f.x * f.y;
            }
            // Every later CTA of the tile starts inside it: the tile is its
            // segment 0.
#pragma unroll 1
            for (int c = first + 1; c <= last; ++c) {
              const size_t off = (size_t)c * g.segs_max * (NB * kTileM) + (size_t)(16 * n16) * kTileM + row;
              const bool in = SEEDLM_IN_BOUNDS(g_check_flag, off + 15 * kTileM, part_n);
              const float* p = partial + (in ? off : 0);
#pragma unroll
              for (int q = 0; q < 16; ++q) v[q] += __ldcg(p + q * kTileM);
            }
            if (gr < g.rows) {
#pragma unroll
              for (int q = 0; q < 16; ++q)
                if (16 * n16 + q < g.M &&
                    SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(16 * n16 + q) * g.rows + gr, y_n))
                  Y[(size_t)(16 * n16 + q) * g.rows + gr] = v[q];
            }
          }
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(dfree(db));
          if (leader && SEEDLM_IN_BOUNDS(g_check_flag, tile, g.tiles)) counters[tile] = 0u;
          return;
        }
      }
      ok = tc::mbar_wait_or_abort(dfull(db), (seg / NACC) & 1, kWaitLimit, abort_flag) && ok;
      tc::fence_after_sync();
#pragma unroll(NB > 64 ? 2 : 4)
      for (int n16 = 0; n16 < NB / 16; ++n16) {
        float v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(32 * eq) << 16) + L::D_COL + ACC * db + 16 * n16, v);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 f = ys[16 * n16 + q];
          v[q] = v[q] * f.x * f.y;
        }
        if (first == last) {
          if (gr < g.rows) {
#pragma unroll
            for (int q = 0; q < 16; ++q)
              if (16 * n16 + q < g.M &&
                  SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(16 * n16 + q) * g.rows + gr, y_n))
                Y[(size_t)(16 * n16 + q) * g.rows + gr] = v[q];
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q)
            if (SEEDLM_IN_BOUNDS(g_check_flag, seg, g.segs_max) &&
                SEEDLM_IN_BOUNDS(g_check_flag, mine_off + (16 * n16 + q) * kTileM + row, part_n))
              mine[(16 * n16 + q) * kTileM + row] = v[q];
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(dfree(db));
      if (first == last) return;
      // The leader publishes the four warps' partial tile (the barrier orders
      // their stores before its fence) and counts it; the last CTA of the
      // tile to count reads every partial after its own fence and barrier.
      tc::named_sync(128);
      if (leader) {
        __threadfence();
        const bool is_last = SEEDLM_IN_BOUNDS(g_check_flag, tile, g.tiles) &&
                             atomicAdd(&counters[tile], 1u) == (unsigned)(last - first);
        if (is_last) __threadfence();
        slot[1] = is_last ? 1u : 0u;
      }
      tc::named_sync(128);
      if (slot[1]) {
        if (gr < g.rows) {
          // Y = partial(first) + partial(first + 1) + ... in CTA order, 16
          // batch rows at a time in registers (independent loads; Y written
          // once).
#pragma unroll 1
          for (int n16 = 0; n16 < NB / 16; ++n16) {
            float acc[16];
#pragma unroll 1
            for (int c = first; c <= last; ++c) {
              const int cseg = tile - (int)(unit_begin(c, g.units, ctas) / g.nchunks);
              const size_t off = ((size_t)c * g.segs_max + cseg) * (NB * kTileM) +
                                 (size_t)(16 * n16) * kTileM + row;
              const bool in = SEEDLM_IN_BOUNDS(g_check_flag, cseg, g.segs_max) &&
                              SEEDLM_IN_BOUNDS(g_check_flag, off + 15 * kTileM, part_n);
              const float* p = partial + (in ? off : 0);
              if (c == first) {
#pragma unroll
                for (int q = 0; q < 16; ++q) acc[q] = __ldcg(p + q * kTileM);
              } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) acc[q] += __ldcg(p + q * kTileM);
              }
            }
#pragma unroll
            for (int q = 0; q < 16; ++q)
              if (16 * n16 + q < g.M &&
                  SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(16 * n16 + q) * g.rows + gr, y_n))
                Y[(size_t)(16 * n16 + q) * g.rows + gr] = acc[q];
          }
        }
        if (leader) counters[tile] = 0u;
      }
      tc::named_sync(128);  // slot[1] is rewritten by the next segment
    };
    UnitCursor ec = c0;
    int seg = 0;
    for (int i = 0; i < n_units; ++i, ec.next(g.nchunks))
      if (i == n_units - 1 || ec.chunk == g.nchunks - 1) epilogue(seg++, ec.tile, i == n_units - 1);
  } else {
    // ------------------------------------------------ producers
    auto produce = [&](int i, const RecUnit<C>& cur) {
      const int as = i % AS;
      if (i >= AS) ok = tc::mbar_wait_or_abort(afree(as), ((i / AS) - 1) & 1, kWaitLimit, abort_flag) && ok;
      tc::fence_after_sync();
      // The thread's BPT * C weights are BPT * C / 2 packed columns of each piece.
      constexpr int NPACK = BPT * C / 2;
      const uint32_t col0 = tmem + ((uint32_t)(32 * lq) << 16) + as * L::STAGE_COLS + kq * NPACK;
      if constexpr (C == 8) {
        // Two blocks at a time: 2^6 W exactly in fp32 (one packed add per
        // pair), then split and stored by one asm statement (eight packed
        // columns of each piece).  The split there -- fp16 truncation and a
        // mixed-precision FMA -- measured 0-3 % faster than masking in fp32.
        constexpr int SB = 2;
#pragma unroll
        for (int j2 = 0; j2 < BPT; j2 += SB) {
          float wv[8 * SB];
#pragma unroll
          for (int jj = 0; jj < SB; ++jj) {
            const BlockC8 blk = rep::decode_c8_rep<kShift>(cur.r[j2 + jj], lane4, lane8);
            const float2 nm = make_float2(__uint_as_float(blk.negm), __uint_as_float(blk.negm));
            w64_pair<0>(blk, nm, wv + 8 * jj);
            w64_pair<2>(blk, nm, wv + 8 * jj);
            w64_pair<4>(blk, nm, wv + 8 * jj);
            w64_pair<6>(blk, nm, wv + 8 * jj);
          }
          tc::tmem_st_f16_split_x8(col0 + 4 * j2, col0 + L::PIECE_COLS + 4 * j2, wv);
        }
      } else {
        uint32_t ph[NPACK], pl[NPACK];
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          const BlockC12 blk = rep::decode_c12_rep<kShift>(cur.r[j], (j ? cur.e >> 4 : cur.e) & 15u, lane8);
          const float2 nm = make_float2(__uint_as_float(blk.negm), __uint_as_float(blk.negm));
          fp16_pieces(weight_bits_c12<0>(blk), weight_bits_c12<1>(blk), nm, neg1, ph[6 * j + 0], pl[6 * j + 0]);
          fp16_pieces(weight_bits_c12<2>(blk), weight_bits_c12<3>(blk), nm, neg1, ph[6 * j + 1], pl[6 * j + 1]);
          fp16_pieces(weight_bits_c12<4>(blk), weight_bits_c12<5>(blk), nm, neg1, ph[6 * j + 2], pl[6 * j + 2]);
          fp16_pieces(weight_bits_c12<6>(blk), weight_bits_c12<7>(blk), nm, neg1, ph[6 * j + 3], pl[6 * j + 3]);
          fp16_pieces(weight_bits_c12<8>(blk), weight_bits_c12<9>(blk), nm, neg1, ph[6 * j + 4], pl[6 * j + 4]);
          fp16_pieces(weight_bits_c12<10>(blk), weight_bits_c12<11>(blk), nm, neg1, ph[6 * j + 5], pl[6 * j + 5]);
        }
        if constexpr (NPACK % 4 == 0) {  // two blocks: 12 columns from a multiple of 4
#pragma unroll
          for (int q = 0; q < NPACK / 4; ++q) {
            tc::tmem_st4(col0 + 4 * q, ph + 4 * q);
            tc::tmem_st4(col0 + L::PIECE_COLS + 4 * q, pl + 4 * q);
          }
        } else {  // one block: 6 columns from an even column
          static_assert(NPACK == 6, "one 12-weight block");
#pragma unroll
          for (int q = 0; q < NPACK / 2; ++q) {
            tc::tmem_st2(col0 + 2 * q, ph + 2 * q);
            tc::tmem_st2(col0 + L::PIECE_COLS + 2 * q, pl + 2 * q);
          }
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(afull(as));
    };

    for (int i0 = 0; i0 < n_units; i0 += kRecAhead) {
#pragma unroll
      for (int k = 0; k < kRecAhead; ++k) {
        const int i = i0 + k;
        if (i < n_units) {
          const RecUnit<C> cur = ring[k];
          if (i + kRecAhead < n_units) {
            load_rec(rc, ring[k]);
            rc.next(g.nchunks);
          }
          produce(i, cur);
        }
      }
    }
  }

  if (!ok) atomicOr(&g_tc_error, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Batch rows of a pass of M rows: M rounded up to 16 up to 64, then 128 or 256.
int nb_of(int M) { return M <= 64 ? (M + 15) / 16 * 16 : (M <= 128 ? 128 : 256); }

int kc_of(int C, int NB) {
  if (C == 8) return NB > 128 ? TcCfg<8, 256>::KC : TcCfg<8, 64>::KC;
  return NB > 128 ? TcCfg<12, 256>::KC : TcCfg<12, 64>::KC;
}

TcGeom make_tc_geom(const seedlm_format& f, int M, const DeviceInfo& dev, int* ctas) {
  TcGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.M = M;
  const int KC = kc_of(f.C, nb_of(M));
  g.nchunks = (f.cols + KC - 1) / KC;
  g.tiles = (f.rows + kTileM - 1) / kTileM;
  g.units = (long long)g.tiles * g.nchunks;
  const int G = g.units < dev.num_sms ? (int)g.units : dev.num_sms;
  int segs = 1;
  for (int b = 0; b < G; ++b) {
    const long long a = (long long)b * g.units / G, e = (long long)(b + 1) * g.units / G;
    const int s = (int)((e - 1) / g.nchunks - a / g.nchunks) + 1;
    if (s > segs) segs = s;
  }
  g.segs_max = segs;
  *ctas = G < 1 ? 1 : G;
  return g;
}

// Workspace: [tile counters][row scale factors][X slabs][partial tiles], each
// part 256-aligned.
struct TcWorkspace {
  int64_t cnt_bytes, scale_bytes, xs_bytes, part_bytes;
  int64_t total() const { return cnt_bytes + scale_bytes + xs_bytes + part_bytes; }
};

int64_t round256(int64_t v) { return (v + 255) / 256 * 256; }

TcWorkspace tc_workspace(const TcGeom& g, int C, int ctas) {
  const int NB = nb_of(g.M);
  TcWorkspace w;
  w.cnt_bytes = round256((int64_t)g.tiles * 4);
  w.scale_bytes = round256((int64_t)NB * 8);
  w.xs_bytes = round256((int64_t)g.nchunks * NB * kc_of(C, NB) * 2);
  w.part_bytes = round256((int64_t)ctas * g.segs_max * NB * kTileM * 4);
  return w;
}

template <int C, int NB>
int launch_tc(const TcGeom& g, int ctas, const uint32_t* rec, const uint8_t* eplane,
              const uint16_t* X, int is_bf16, float* Y, unsigned char* ws, const TcWorkspace& w,
              cudaStream_t stream, const DeviceInfo& dev) {
  using L = TcSmem<C, NB>;
  if ((size_t)L::TOTAL > (size_t)dev.max_smem_optin) return SEEDLM_EUNSUPPORTED;
  int rc = allow_max_smem((const void*)gemm_tc_kernel<C, NB>, dev);
  if (rc) return rc;
  unsigned int* counters = reinterpret_cast<unsigned int*>(ws);
  float2* yscale = reinterpret_cast<float2*>(ws + w.cnt_bytes);
  unsigned char* xs = ws + w.cnt_bytes + w.scale_bytes;
  float* partial = reinterpret_cast<float*>(ws + w.cnt_bytes + w.scale_bytes + w.xs_bytes);

  // stage_x: NB rows x parts CTAs, about 256 column groups of 8 per CTA (at
  // most 64 parts).  For bf16 X every CTA reads its whole row for the
  // maximum unless the row's parts form a cluster; measured, the cluster
  // pays from 5 parts on (8192 x 28672, M = 64: 140 -> 135 us) and costs
  // about 1 us below (28672 x 8192, 4 parts), so wide rows take clusters of
  // up to 8 parts (the portable size) and the rest the plain launch.
  const int groups = g.nchunks * (L::KC / 8);
  int parts = groups / 256 < 1 ? 1 : (groups / 256 > 64 ? 64 : groups / 256);
  const bool cluster = is_bf16 && parts > 4;
  if (cluster && parts > 8) parts = 8;
  const int vec = (reinterpret_cast<uintptr_t>(X) % 16 == 0) && (g.cols % 8 == 0);
  {
    cudaLaunchConfig_t scfg = {};
    scfg.gridDim = dim3(NB * parts);
    scfg.blockDim = dim3(256);
    scfg.stream = stream;
    cudaLaunchAttribute sattr[1];
    sattr[0].id = cudaLaunchAttributeClusterDimension;
    sattr[0].val.clusterDim.x = cluster ? parts : 1;
    sattr[0].val.clusterDim.y = 1;
    sattr[0].val.clusterDim.z = 1;
    scfg.attrs = sattr;
    scfg.numAttrs = 1;
    const cudaError_t serr = cudaLaunchKernelEx(&scfg, stage_x_kernel<L::KC, NB>, X, g.M, g.cols,
                                                g.nchunks, is_bf16, (int)cluster, parts, vec, xs,
                                                yscale);
    if (serr != cudaSuccess) return record_cuda_error(serr);
  }
  count_launch();
  if ((rc = record_cuda_error(cudaGetLastError()))) return rc;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(Roles<C>::kThreads);
  cfg.dynamicSmemBytes = L::TOTAL;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<C, NB>, rec, eplane,
                                       (const unsigned char*)xs, (const float2*)yscale, Y, partial,
                                       counters, g);
  if (err != cudaSuccess) return record_cuda_error(err);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

template <int C>
int dispatch_nb(const TcGeom& g, int ctas, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* X, int is_bf16, float* Y, unsigned char* ws, const TcWorkspace& w,
                cudaStream_t st, const DeviceInfo& dev) {
  switch (nb_of(g.M)) {
    case 16: return launch_tc<C, 16>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
    case 32: return launch_tc<C, 32>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
    case 48: return launch_tc<C, 48>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
    case 64: return launch_tc<C, 64>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
    case 128: return launch_tc<C, 128>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
    default: return launch_tc<C, 256>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
  }
}

int dispatch_tc(const seedlm_format& f, const TcGeom& g, int ctas, const uint32_t* rec,
                const uint8_t* eplane, const uint16_t* X, int is_bf16, float* Y,
                unsigned char* ws, const TcWorkspace& w, cudaStream_t st, const DeviceInfo& dev) {
  if (f.C == 8) return dispatch_nb<8>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
  return dispatch_nb<12>(g, ctas, rec, eplane, X, is_bf16, Y, ws, w, st, dev);
}

}  // namespace

int64_t gemm_tc_workspace_bytes(const seedlm_format& f, int M, const DeviceInfo& dev) {
  int ctas = 1;
  const TcGeom g = make_tc_geom(f, M, dev, &ctas);
  return tc_workspace(g, f.C, ctas).total();
}

int launch_gemm_tc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                   const uint16_t* X, int is_bf16, int M, float* Y, void* workspace,
                   int64_t workspace_bytes, cudaStream_t stream, const DeviceInfo& dev) {
  int ctas = 1;
  const TcGeom g = make_tc_geom(f, M, dev, &ctas);
  const TcWorkspace w = tc_workspace(g, f.C, ctas);
  if (workspace_bytes < w.total()) return SEEDLM_EINVAL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SEEDLM_EINVAL;
  return dispatch_tc(f, g, ctas, rec, eplane, X, is_bf16, Y,
                     static_cast<unsigned char*>(workspace), w, stream, dev);
}

namespace {

// A bounded mbarrier wait that nothing ends: the same wait, give-up flag and
// TMEM handling as gemm_tc_kernel, run on purpose into its time limit.
__global__ void __launch_bounds__(64, 1) wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t slot[3];
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(&bar), 1);  // one arrival expected, none will come
    tc::fence_mbar_init();
    slot[2] = 0u;
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(slot), 32);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const bool ok = tc::mbar_wait_or_abort(tc::smem_u32(&bar), 0, limit_ns, slot + 2);
  if (!ok && threadIdx.x == 0) atomicOr(&g_tc_error, 1u);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(slot[0], 32);
  }
}

// One bounds check evaluated on the device, with no memory access behind it:
// shows that a checked build's comparison and flag reach seedlm_device_error.
__global__ void bounds_check_kernel(long long index, long long extent) {
  if (SEEDLM_IN_BOUNDS(g_check_flag, index, extent)) {
  }
}

}  // namespace

int launch_bounds_check(int64_t index, int64_t extent, cudaStream_t stream) {
  bounds_check_kernel<<<1, 1, 0, stream>>>(index, extent);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

int launch_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 64, 0, stream>>>(limit_ns);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

int read_and_clear_tc_error(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v));
  if (err != cudaSuccess) return record_cuda_error(err);
  if (v) {
    err = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
    if (err != cudaSuccess) return record_cuda_error(err);
  }
  *out = v;
  return SEEDLM_OK;
}

// ------------------------------------------------ allocation-free variant
//
// For callers that cannot allocate device memory themselves, the workspace of
// the tensor-core GEMM (tile counters, X slabs, partial tiles) lives in one
// array that the library owns for the life of the process.

constexpr int64_t kNoAllocBytes = (16ll << 20) + (64ll << 10);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device (the name is only
// a host-side stand-in for it).  Outside a stream capture it is looked up on
// every call, so a context that was reset and reloaded the module is seen;
// during a capture the address found by an earlier call on this device is
// used (a lookup there could load the module inside the capture), and there
// must have been one.
int noalloc_scratch(const DeviceInfo& dev, cudaStream_t st, unsigned char** out) {
  if (dev.device < 0 || dev.device >= 64) return SEEDLM_EUNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t err = cudaStreamIsCapturing(st, &cap);
  if (err != cudaSuccess) return record_cuda_error(err);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return record_cuda_error(err);
    if (!p) return SEEDLM_ECUDA;
    g_noalloc_addr[dev.device] = p;
  } else if (!g_noalloc_addr[dev.device]) {
    return SEEDLM_EUNSUPPORTED;  // first call on this device inside a capture
  }
  *out = static_cast<unsigned char*>(g_noalloc_addr[dev.device]);
  return SEEDLM_OK;
}

}  // namespace

}  // namespace seedlm

using namespace seedlm;

extern "C" SEEDLM_API int seedlm_gemm_smallM_noalloc(const seedlm_format* fmt,
                                                     const uint32_t* rec, const uint8_t* eplane,
                                                     const void* X, int x_dtype, int M, float* Y,
                                                     seedlm_stream stream) {
  int rc = check_format(fmt);
  if (rc) return rc;
  if ((rc = check_planes(fmt, rec, eplane))) return rc;
  if (x_dtype != SEEDLM_F16 && x_dtype != SEEDLM_BF16) return SEEDLM_EINVAL;
  if (M < 1 || M > 64) return SEEDLM_EINVAL;
  if (fmt->rows == 0) return SEEDLM_OK;
  if (!Y || !aligned(Y, 4)) return SEEDLM_EINVAL;
  if (fmt->cols > 0 && (!X || !aligned(X, 2))) return SEEDLM_EINVAL;
  DeviceInfo dev;
  if ((rc = current_device_info(&dev))) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if (fmt->cols == 0)
    return record_cuda_error(cudaMemsetAsync(Y, 0, (size_t)M * fmt->rows * sizeof(float), st));
  const uint16_t* Xh = static_cast<const uint16_t*>(X);
  const int is_bf16 = x_dtype == SEEDLM_BF16;
  if (M == 1 && gemv_smem_bytes(*fmt, dev) > 0)
    return launch_gemv(*fmt, rec, eplane, Xh, is_bf16, Y, st, dev);
  if (gemm_cc_applies(*fmt, M)) return launch_gemm_cc(*fmt, rec, eplane, Xh, is_bf16, M, Y, st, dev);

  int ctas = 1;
  const TcGeom g = make_tc_geom(*fmt, M, dev, &ctas);
  const TcWorkspace w = tc_workspace(g, fmt->C, ctas);
  if (w.total() > kNoAllocBytes) return SEEDLM_EUNSUPPORTED;  // needs more than the library holds
  unsigned char* base = nullptr;
  if ((rc = noalloc_scratch(dev, st, &base))) return rc;
  // The counters must start at zero; the last call may have left them in any
  // state if it failed part-way.
  if ((rc = record_cuda_error(cudaMemsetAsync(base, 0, (size_t)w.cnt_bytes, st)))) return rc;
  return dispatch_tc(*fmt, g, ctas, rec, eplane, Xh, is_bf16, Y, base, w, st, dev);
}
