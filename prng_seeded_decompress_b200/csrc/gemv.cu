// gemv.cu -- y = W x with W rebuilt block by block on the fly (batch 1).
//
// SeedLM inference (paperhub.cn review thread, authors' reply on how inference
// uses Eq (1)): the seed and coefficients of each block are read from memory,
// the block is rebuilt and consumed at once; W never exists in full precision.
//
// On B200 this product is bound by the SM, not by HBM: a 4-bit block of 8
// weights costs 16 dp2a, 8 funnel shifts and 8 packed fp32 operations of
// arithmetic (seedlm_device.cuh) plus its decode, and the decode's table
// lookups are random.  The kernel is organised around two facts:
//
//   * Lane-replicated tables, conflict-free, at fixed shared addresses
//     (rep_tables.cuh): one shared-memory wavefront per lookup instead of
//     ~3.2 for random indices into a single copy, which saturated the
//     shared-memory pipe before, and a one-instruction address (one prmt of
//     the record's index byte next to the lane's offset; the table base
//     rides in the load's immediate offset).  The dynamic shared allocation
//     must start at shared address kSmemBase for this (checked at entry; a
//     mismatch raises the device error flag and the kernel does nothing).
//
// Work decomposition (one CTA per SM, persistent):
//   * x is converted to fp32 into shared memory in a swizzled "record pair"
//     layout: for records 2rp and 2rp+1 of a row the x values of column c of
//     both blocks sit side by side, so one packed fp32x2 FMA consumes weight
//     c of both blocks.  x is staged in column segments of at most
//     kMaxSegSpans<C> spans (32 record pairs each), so any width works.
//   * An item is a group of 4 rows x one span of 32 record pairs (one pair
//     per lane): the lane loads the two records of each row (8 bytes,
//     coalesced across the warp), keeps the pair's x values in registers for
//     all 4 rows, and accumulates one fp32x2 sum per row.  Record sets are
//     loaded ahead of the one being rebuilt.
//   * Each CTA owns a contiguous range of row groups and splits the items of
//     each (pass, segment) evenly over its warps.  Row sums are reduced with
//     warp shuffles and added into a per-warp slot in shared memory; after a
//     barrier the slots of each row are added in warp order -- the same
//     order on every call -- and written.
//   * Launched with programmatic stream serialization, and every CTA lets
//     the next kernel launch as soon as it starts: a CTA of the next GEMV
//     takes its SM when this one's CTA there exits and fills its tables
//     (before griddepcontrol.wait) while the slowest CTAs of this grid
//     finish.  Records and x are read only after the wait, so they may be
//     written by the previous kernel in the stream.
#include <cuda_runtime.h>

#include <type_traits>

#include "rep_tables.cuh"
#include "seedlm_device.cuh"
#include "seedlm_internal.h"

// Float operations per pair of weights (one in each of the lane's two
// blocks): 0 = one packed fp32x2 add (int -> float) + one packed fp32x2 FMA;
// 1 = two scalar adds + one packed FMA (moves the adds off the pipe the dp2a
// instructions use).
#ifndef SEEDLM_GEMV_FP_MODE
#define SEEDLM_GEMV_FP_MODE 0
#endif

// How a C = 8 block gets its stream bits 16..47 (the LFSR states past the
// seed).  The pages name the LFSR as the generator and note that GPUs lack
// hardware for it (paperhub.cn review thread, authors' reply on GPU
// implementation challenges); three ways to run it on the SM:
//   0 = GF(2) jump tables: two lane-replicated 256-entry tables indexed by
//       the seed's bytes, xor-ed (the library's choice);
//   1 = register stepping: the recurrence b[m+16] = b[m]^b[m+2]^b[m+3]^b[m+5]
//       applied to 32-bit words, three passes of shifts and xors;
//   2 = one table of the whole 65,535-state cycle: records then hold the
//       seed's position in the cycle instead of the seed (a one-time
//       relabelling, a bijection), and a block's window is one 8-byte load
//       at that position.  For comparisons only: the library's record format
//       stores seeds, so this build does not compute the library's product.
#ifndef SEEDLM_GEMV_LFSR
#define SEEDLM_GEMV_LFSR 0
#endif

// Record sets in flight ahead of the one being rebuilt, C = 8.
#ifndef SEEDLM_GEMV_PREFETCH8
#define SEEDLM_GEMV_PREFETCH8 1
#endif

// Blocks per lane and row for C = 8 (2 or 4); see Tune below.
#ifndef SEEDLM_GEMV_BPL8
#define SEEDLM_GEMV_BPL8 4
#endif

namespace seedlm {

SEEDLM_CHECK_FLAG(gemv)

namespace {

__device__ unsigned int g_gemv_error = 0;

// Blocks of one row a lane takes per item (one 8- or 16-byte record load),
// warps per CTA (one CTA per SM) and record sets in flight ahead of the one
// being rebuilt.  C = 8 takes 4 blocks (a quad) per lane and row, so the
// per-item work (addresses, loads, loop) is spread over 16 blocks; with 32
// x values per lane that needs the register file of 16 warps.  C = 12 takes
// 2 blocks (a pair): its four dp2a windows per weight already fill 128
// registers.
template <int C, int V>
struct Tune {
  static constexpr int kBPL = (C == 8 && V == 0) ? SEEDLM_GEMV_BPL8 : 2;
  static constexpr int kWarps = (V == 1) ? 8 : (C == 8 && kBPL == 2) ? 24 : 16;
  static constexpr int kPrefetch = (C == 8) ? SEEDLM_GEMV_PREFETCH8 : 2;
  static constexpr int kMinBlocks = (V == 1) ? 2 : 1;  // CTAs per SM the launch bounds ask for
};
constexpr int kRowsPerTask = 4;
constexpr int kMinWarps = 8;      // warps per CTA however few items it has
constexpr int kSpanUnits = 32;    // lane units (pairs or quads of blocks) per span

// V = 2 is V = 0 with half-warp spans: each half-warp takes 16 units of its
// own 4 rows, so an item is 8 rows x 16 units.  Chosen where it pads a row's
// units less (3-bit rows of 4096 columns: 171 pairs fill 176 lanes instead
// of 192).
template <int V>
__host__ __device__ constexpr int span_units() { return V == 2 ? kSpanUnits / 2 : kSpanUnits; }
template <int V>
__host__ __device__ constexpr int rows_per_item() { return kRowsPerTask * (kSpanUnits / span_units<V>()); }

// Two variants of the kernel:
//   V = 0 (large products): the lane-replicated tables at absolute shared
//     addresses, one CTA per SM.  Shared-memory map:
//       C = 8:  [kSmemBase, 0x10000)  x slots of one column segment
//               [0x10000, 0x20000)    stream jump-table rows
//               [0x20000, 0x30000)    coefficient-table rows
//       C = 12: [kSmemBase, 0x20000)  x slots of one column segment
//               [0x20000, 0x30000)    stream jump-table rows
//       both:   [0x30000, ...)        partial row sums of one pass
//   V = 2: V = 0 with half-warp spans (above), for C = 12.
//   V = 1 (small products, a few items per CTA): one copy of each table at
//     the start of the allocation, 32 KB of x slots after it, then the
//     partial sums; 8 warps and small allocations, so that several CTAs --
//     of this launch and of the next one in the stream -- share an SM.  On
//     a 512 x 512 matrix the replicated tables' setup (128 KB of shared
//     stores, one CTA per SM) costs more than the product itself.
using rep::kSmemBase;
using rep::lds32;
using rep::lds64;
template <int C, int V>
struct Smem {
  static constexpr uint32_t kJump = rep::tables_begin<C>();  // V = 0, 2
  // V = 1: jump tables (C = 8: 2 x 256 words; C = 12: 2 x 256 8-byte
  // entries) then, for C = 8, the two coefficient tables (2 x 256 x 8 B).
  static constexpr int kTabBytes = (V != 1) ? 0 : (C == 8) ? 2048 + 4096 : 4096;
  static constexpr int kXOff = kTabBytes;  // bytes from the allocation's start
  static constexpr int kXBytes = (V != 1) ? (int)(kJump - kSmemBase) : 32768;
  static constexpr int kPartOff = (V != 1) ? (int)(0x30000u - kSmemBase) : kXOff + kXBytes;
  // x floats per lane unit: C * kBPL, rounded up to 32 for C = 12 (swizzle).
  static constexpr int kSlotFloats = (C == 8) ? 8 * Tune<C, V>::kBPL : 32;
  static constexpr int kSpanBytes = span_units<V>() * kSlotFloats * 4;
  static constexpr int kMaxSegSpans = kXBytes / kSpanBytes;
  static constexpr int kPartBytesPerGroup = rows_per_item<V>() * 4;  // per warp
};
#if SEEDLM_GEMV_LFSR == 2
constexpr uint32_t kTabJump = Smem<8, 0>::kJump;
#endif

struct GemvGeom {
  int rows, cols, nb, rec_pitch, e_pitch;
  int n_spans;      // ceil(ceil(nb / kBPL) / span units)
  int groups;       // ceil(rows / rows per item)
  int full_groups;  // groups with all their rows inside the matrix
  int full_spans;   // spans whose every unit lies inside the row pitch
  int seg_spans;    // spans per x segment (the last one may be shorter)
  int n_segs;
  int pass_groups;  // row groups per partial-sum pass
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

#if SEEDLM_GEMV_LFSR == 1
// One pass of the recurrence on a 32-bit word X whose bits [0, n) are stream
// bits [0, n): bit m of the result is stream bit 16 + m for m + 5 < n.
// x>>3 ^ x>>5 = (x ^ x>>2) >> 3, so a pass is two shift-xor pairs.
__device__ __forceinline__ uint32_t lfsr_pass(uint32_t x) {
  const uint32_t u = x ^ (x >> 2);
  return u ^ (u >> 3);
}
#endif

#if SEEDLM_GEMV_LFSR == 2
// Seed at positions 0, 8, 16, ... of the cycle that starts at seed 1.
struct CycleSeeds {
  uint16_t s[8192];
};
constexpr CycleSeeds make_cycle_seeds() {
  CycleSeeds t{};
  uint32_t st = 1;
  for (int p = 0; p < 8192 * 8; ++p) {
    if ((p & 7) == 0) t.s[p >> 3] = (uint16_t)st;
    const uint32_t bit = (st ^ (st >> 2) ^ (st >> 3) ^ (st >> 5)) & 1u;
    st = (st >> 1) | (bit << 15);
  }
  return t;
}
__device__ const CycleSeeds kCycleSeeds = make_cycle_seeds();
#endif

// Fills the decode tables: for V = 1 one copy of each at the start of the
// allocation, for V = 0 the lane-replicated rows (rep_tables.cuh).
template <int C, int V>
__device__ void fill_tables(unsigned char* smem) {
  if constexpr (V == 1) {
    // One copy: C = 8 words t_lo[256], t_hi[256], then tq1[256], tq2[256]
    // (fill_coef_tables_c8's layout); C = 12 8-byte t_lo[256], t_hi[256].
    for (int i = threadIdx.x; i < 512; i += blockDim.x) {
      const uint64_t e = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
      if constexpr (C == 8)
        reinterpret_cast<uint32_t*>(smem)[i] = (uint32_t)e;
      else
        reinterpret_cast<uint2*>(smem)[i] = make_uint2((uint32_t)e, (uint32_t)(e >> 32));
    }
    if constexpr (C == 8) {
      // The layout decode_c8_tab reads (it adds bits(M) itself).
      uint2* tq = reinterpret_cast<uint2*>(smem + 2048);
      fill_coef_tables_c8(tq, tq + 256, threadIdx.x, blockDim.x);
    }
    return;
  }
  rep::fill_rep_tables<C, 0>(smem, threadIdx.x, blockDim.x);
#if SEEDLM_GEMV_LFSR == 2
  if constexpr (C == 8) {
    // Cycle-window table: entry k = the seed at position 8k followed by its
    // stream bits 16..63, written over the jump rows (64 KB).
    __syncthreads();
    uint2* cw = reinterpret_cast<uint2*>(smem + (Smem<C, 0>::kJump - kSmemBase));
    for (int i = threadIdx.x; i < 8192; i += blockDim.x) {
      const uint32_t sd = kCycleSeeds.s[i];
      const uint64_t ext = kStreamTables.lo[sd & 0xffu] ^ kStreamTables.hi[sd >> 8];
      const uint64_t e = (uint64_t)sd | (ext << 16);
      cw[i] = make_uint2((uint32_t)e, (uint32_t)(e >> 32));
    }
  }
#endif
}

// C = 8 decode from the replicated tables (rep_tables.cuh), or by one of the
// comparison LFSR variants.
__device__ __forceinline__ BlockC8 decode_c8_rep(uint32_t rec, uint32_t lane4, uint32_t lane8) {
#if SEEDLM_GEMV_LFSR == 0
  return rep::decode_c8_rep<0>(rec, lane4, lane8);
#else
  BlockC8 b;
#if SEEDLM_GEMV_LFSR == 1
  b.lo = rec;
  // Passes over 16, 27 and 32 valid stream bits: stream bits 16..42.
  const uint32_t t1 = lfsr_pass(rec);                     // bits 16..26 valid at 16..26
  const uint32_t t2 = lfsr_pass(prmt<0x7632u>(rec, t1));  // stream 0..26 -> 16..37 at 0..21
  b.hi = lfsr_pass(prmt<0x5432u>(rec, t2));               // stream 0..31 -> 16..42 at 0..26
#else
  // rec bits [16,32) = position P in the cycle; the table entry k holds
  // cycle bits [8k, 8k + 64).
  const uint32_t pos = rec >> 16;
  const uint2 w = lds64<kTabJump>(pos & 0xfff8u);
  const uint32_t sh = pos & 7u;
  const uint32_t s_lo = __funnelshift_r(w.x, w.y, sh), s_hi = w.y >> sh;  // bits [P, P+56)
  b.lo = s_lo << 16;
  b.hi = __funnelshift_r(s_lo, s_hi, 16);
#endif
  const uint2 c1 = lds64<rep::kCoef8>(prmt<0x5504u>(rec, lane8));
  const uint2 c2 = lds64<rep::kCoef8 + 128>(prmt<0x5514u>(rec << 4, lane8));
  b.a01 = c1.x;
  b.a23 = c2.x;
  const uint32_t e23 = (rec << 11) & 0x07800000u;  // e << 23
  b.init = (int32_t)(c1.y + c2.y - e23);
  b.negm = kNegMagicBits - e23;
  return b;
#endif
}

__device__ __forceinline__ BlockC12 decode_c12_rep(uint32_t rec, uint32_t e4, uint32_t lane8) {
  return rep::decode_c12_rep<0>(rec, e4, lane8);
}

// x slot layout, per lane unit u (kBPL consecutive blocks of a row):
//   C = 8, pairs:  16 floats; float4 i holds column 2i and 2i+1 of both
//                  blocks (h = 0, 1 interleaved), at float4 i ^ ((u >> 1) & 3)
//   C = 8, quads:  32 floats; float4 c holds column c of blocks 0..3, at
//                  float4 c ^ (u & 7)
//   C = 12, pairs: 32 floats (24 used); float4 i holds columns 2i, 2i+1 of
//                  both blocks, at float4 i ^ (u & 7)
// so each lane reads its unit with 16-byte loads and one packed fp32x2 FMA
// takes weight c of two blocks; the XOR swizzles keep the 8 lanes of a
// quarter-warp on distinct bank groups.
template <int C, int V>
__device__ __forceinline__ int x_slot_index(int u, int c, int h) {
  if constexpr (C == 8 && Tune<8, V>::kBPL == 4) {
    return u * 32 + ((c ^ (u & 7)) << 2) + h;
  } else if constexpr (C == 8) {
    return u * 16 + (((c >> 1) ^ ((u >> 1) & 3)) << 2) + ((c & 1) << 1) + h;
  } else {
    return u * 32 + (((c >> 1) ^ (u & 7)) << 2) + ((c & 1) << 1) + h;
  }
}

// x columns of spans [s0, s0 + sl), zero past cols, into the segment's
// slots.  One thread per lane unit; 16-byte loads when x is 16-byte aligned
// and the unit lies inside x, and one 16-byte store per float4 of the slot:
// the 8 threads of a quarter-warp then write 8 distinct bank groups (the
// slot swizzle), where scalar stores met 4-way conflicts.
template <int C, int V>
__device__ void stage_x(float* xs, const uint16_t* __restrict__ x, int is_bf16, const GemvGeom& g,
                        int s0, int sl) {
  constexpr int kBPL = Tune<C, V>::kBPL;
  constexpr int kVals = C * kBPL;  // x values of one unit (16, 24 or 32)
  const int units = sl * span_units<V>();
  const int col_base = s0 * span_units<V>() * kVals;
  const bool vec = (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = Smem<C, V>::kXBytes / 4;)
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    const int col0 = col_base + u * kVals;
    uint32_t w[kVals / 2];  // value k in the half k % 2 of w[k / 2]
    if (vec && col0 + kVals <= g.cols) {
#pragma unroll
      for (int k = 0; k < kVals / 8; ++k) {
        const uint4 q = *reinterpret_cast<const uint4*>(x + col0 + 8 * k);
        w[4 * k] = q.x;
        w[4 * k + 1] = q.y;
        w[4 * k + 2] = q.z;
        w[4 * k + 3] = q.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < kVals / 2; ++k) {
        const uint32_t lo = col0 + 2 * k < g.cols ? x[col0 + 2 * k] : 0u;
        const uint32_t hi = col0 + 2 * k + 1 < g.cols ? x[col0 + 2 * k + 1] : 0u;
        w[k] = lo | hi << 16;
      }
    }
    auto val = [&](int k) { return act_to_float((uint16_t)(w[k >> 1] >> (16 * (k & 1))), is_bf16); };
    // float4 i of the slot: column i of blocks 0..3 (quads), or columns 2i,
    // 2i+1 of blocks 0 and 1 (pairs); see x_slot_index.
#pragma unroll
    for (int i = 0; i < kVals / 4; ++i) {
      float4 f;
      int si;
      if constexpr (C == 8 && kBPL == 4) {
        f = make_float4(val(i), val(8 + i), val(16 + i), val(24 + i));
        si = x_slot_index<C, V>(u, i, 0);
      } else {
        f = make_float4(val(2 * i), val(C + 2 * i), val(2 * i + 1), val(C + 2 * i + 1));
        si = x_slot_index<C, V>(u, 2 * i, 0);
      }
      if (SEEDLM_IN_BOUNDS(g_check_flag, si + 3, xs_floats)) *reinterpret_cast<float4*>(xs + si) = f;
    }
  }
}

// The records one lane needs for one (row group, span) item: its unit of
// kBPL blocks in each of the group's 4 rows, plus for C = 12 the exponent
// byte of the pair.  Rows past `rows` and units past the row pitch read as
// zero records (their x is zero, so they add nothing).
template <int C, int V>
struct RecSet {
  using Unit = typename std::conditional<Tune<C, V>::kBPL == 4, uint4, uint2>::type;
  Unit r[kRowsPerTask];
  uint32_t e[C == 12 ? kRowsPerTask : 1];
};

template <int C, int V>
__device__ __forceinline__ void load_unit(typename RecSet<C, V>::Unit& o, const uint32_t* p) {
  if constexpr (Tune<C, V>::kBPL == 4) o = ld_stream_u4(p);
  else o = ld_stream_u2(p);
}

template <int C, int V>
__device__ __forceinline__ void load_set(RecSet<C, V>& o, const uint32_t* __restrict__ rec,
                                         const uint8_t* __restrict__ eplane, const GemvGeom& g,
                                         int grp, int span, int lane) {
  constexpr int kBPL = Tune<C, V>::kBPL;
  constexpr int kSU = span_units<V>();
  const int row0 = grp * rows_per_item<V>() + (lane / kSU) * kRowsPerTask;
  const int u = span * kSU + lane % kSU;
  const uint32_t* p = rec + (size_t)row0 * g.rec_pitch + kBPL * u;
  if (grp < g.full_groups && span < g.full_spans && !SEEDLM_CHECK) {
    // Every row of the group and every unit of the span is inside the plane.
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j) load_unit<C, V>(o.r[j], p + (size_t)j * g.rec_pitch);
  } else {
    const bool unit_ok = kBPL * u < g.rec_pitch;
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j) {
      // The unit's last record is the last word read.
      const bool ok = unit_ok && row0 + j < g.rows &&
                      SEEDLM_IN_BOUNDS(g_check_flag,
                                       (size_t)(row0 + j) * g.rec_pitch + kBPL * u + kBPL - 1,
                                       (size_t)g.rows * g.rec_pitch);
      if (ok) load_unit<C, V>(o.r[j], p + (size_t)j * g.rec_pitch);
      else o.r[j] = typename RecSet<C, V>::Unit{};
    }
  }
  if constexpr (C == 12) {
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j)
      o.e[j] = (row0 + j < g.rows && u < g.e_pitch &&
                SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(row0 + j) * g.e_pitch + u,
                                 (size_t)g.rows * g.e_pitch))
                   ? ld_stream_u8(eplane + (size_t)(row0 + j) * g.e_pitch + u)
                   : 0u;
  }
}

// Record words (32 MiB) from which a 4-bit GEMV prefetches its first record
// sets into L2 before waiting for the previous kernel.
constexpr int64_t kL2PrefetchMinWords = (int64_t)8 << 20;

// L2 prefetch of the record lines load_set would read, for full groups and
// spans only (the addresses the unchecked fast path of load_set reads).
template <int C, int V>
__device__ __forceinline__ void prefetch_set(const uint32_t* __restrict__ rec, const GemvGeom& g,
                                             int grp, int span, int lane) {
  if (grp >= g.full_groups || span >= g.full_spans) return;
  constexpr int kSU = span_units<V>(), kBPL = Tune<C, V>::kBPL;
  const int row0 = grp * rows_per_item<V>() + (lane / kSU) * kRowsPerTask;
  const int u = span * kSU + lane % kSU;
#pragma unroll
  for (int j = 0; j < kRowsPerTask; ++j) {
    const size_t w = (size_t)(row0 + j) * g.rec_pitch + kBPL * u;
    if (SEEDLM_IN_BOUNDS(g_check_flag, w + kBPL - 1, (size_t)g.rows * g.rec_pitch))
      prefetch_l2(rec + w);
  }
}

#ifndef SEEDLM_GEMV_C12_ORDER
#define SEEDLM_GEMV_C12_ORDER 1
#endif


#if SEEDLM_GEMV_C12_ORDER == 1
// Window k (stream bits [k, k+32)) of a C = 12 block holds state k in its
// low half and state k+16 in its high half; state 12p + c belongs to weight
// c with coefficient q_p.  Windows 0..31 cover all 48 states.
template <int k>
__device__ __forceinline__ void c12_windows(const BlockC12& A, const BlockC12& B, int32_t (&va)[12],
                                            int32_t (&vb)[12]) {
  if constexpr (k < 32) {
    const uint32_t wa = window_c12<k>(A), wb = window_c12<k>(B);
    constexpr int lo_p = k / 12, lo_c = k % 12;              // state k
    constexpr int hi_p = (k + 16) / 12, hi_c = (k + 16) % 12;  // state k + 16
    if constexpr (lo_p < 4 && k < 24) {
      va[lo_c] = dp2a_lo_su(A.a[lo_p], wa, va[lo_c]);
      vb[lo_c] = dp2a_lo_su(B.a[lo_p], wb, vb[lo_c]);
    }
    if constexpr (hi_p < 4 && k >= 8) {
      va[hi_c] = dp2a_hi_su(A.a[hi_p], wa, va[hi_c]);
      vb[hi_c] = dp2a_hi_su(B.a[hi_p], wb, vb[hi_c]);
    }
    c12_windows<k + 1>(A, B, va, vb);
  }
}
#endif

// Weight pair (c of block A, c of block B) -> fp32x2, accumulated against
// the pair's x values.
__device__ __forceinline__ float2 fma_pair(int32_t bits_a, int32_t bits_b, float2 negm, float2 xv,
                                           float2 acc) {
#if SEEDLM_GEMV_FP_MODE == 1
  const float2 w = make_float2(__int_as_float(bits_a) + negm.x, __int_as_float(bits_b) + negm.y);
  return __ffma2_rn(w, xv, acc);
#else
  const float2 w = make_float2(__int_as_float(bits_a), __int_as_float(bits_b));
  return __ffma2_rn(__fadd2_rn(w, negm), xv, acc);
#endif
}

// The decode of the variant: replicated tables (V = 0) or the single copies
// at the start of the allocation (V = 1).
template <int V>
__device__ __forceinline__ BlockC8 decode_c8_v(uint32_t rec, uint32_t lane4, uint32_t lane8,
                                               const unsigned char* tabs) {
  if constexpr (V != 1) {
    return decode_c8_rep(rec, lane4, lane8);
  } else {
    const uint32_t* t = reinterpret_cast<const uint32_t*>(tabs);
    const uint2* tq = reinterpret_cast<const uint2*>(tabs + 2048);
    return decode_c8_tab(rec, t, t + 256, tq, tq + 256);
  }
}

template <int V>
__device__ __forceinline__ BlockC12 decode_c12_v(uint32_t rec, uint32_t e4, uint32_t lane8,
                                                 const unsigned char* tabs) {
  if constexpr (V != 1) {
    return decode_c12_rep(rec, e4, lane8);
  } else {
    const uint2* t = reinterpret_cast<const uint2*>(tabs);
    return decode_c12(rec, e4, t, t + 256);
  }
}

// Blocks A and B of one row (x pairs xv[c] = (x of A's column c, x of B's)).
template <int V>
__device__ __forceinline__ float2 dot_c8(uint32_t ra, uint32_t rb, const float2 (&xv)[8],
                                         uint32_t lane4, uint32_t lane8,
                                         const unsigned char* tabs, float2 a) {
  const BlockC8 A = decode_c8_v<V>(ra, lane4, lane8, tabs);
  const BlockC8 B = decode_c8_v<V>(rb, lane4, lane8, tabs);
  const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
#define SEEDLM_C8_STEP(c) a = fma_pair(weight_bits_c8<c>(A), weight_bits_c8<c>(B), negm, xv[c], a);
  SEEDLM_C8_STEP(0) SEEDLM_C8_STEP(1) SEEDLM_C8_STEP(2) SEEDLM_C8_STEP(3)
  SEEDLM_C8_STEP(4) SEEDLM_C8_STEP(5) SEEDLM_C8_STEP(6) SEEDLM_C8_STEP(7)
#undef SEEDLM_C8_STEP
  return a;
}

// Rebuild the lane's kBPL x C weights of each of the 4 rows and accumulate
// w * x into one fp32x2 sum per row.  ul is the lane's unit within the
// staged segment.
template <int C, int V>
__device__ __forceinline__ void rebuild_and_dot(const RecSet<C, V>& cur,
                                                const float* __restrict__ xs, int ul, int lane,
                                                uint32_t lane4, uint32_t lane8,
                                                const unsigned char* tabs,
                                                float2 (&acc)[kRowsPerTask]) {
  const float* slot = xs + ul * Smem<C, V>::kSlotFloats;
  if constexpr (C == 8 && Tune<8, V>::kBPL == 4) {
    const int swz = lane & 7;
    float2 x01[8], x23[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 v = *reinterpret_cast<const float4*>(slot + ((c ^ swz) << 2));
      x01[c] = make_float2(v.x, v.y);
      x23[c] = make_float2(v.z, v.w);
    }
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j) {
      float2 a = dot_c8<V>(cur.r[j].x, cur.r[j].y, x01, lane4, lane8, tabs, acc[j]);
      acc[j] = dot_c8<V>(cur.r[j].z, cur.r[j].w, x23, lane4, lane8, tabs, a);
    }
  } else if constexpr (C == 8) {
    const int swz = (lane >> 1) & 3;
    float2 xp[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = *reinterpret_cast<const float4*>(slot + ((i ^ swz) << 2));
      xp[2 * i] = make_float2(v.x, v.y);
      xp[2 * i + 1] = make_float2(v.z, v.w);
    }
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j)
      acc[j] = dot_c8<V>(cur.r[j].x, cur.r[j].y, xp, lane4, lane8, tabs, acc[j]);
  } else {
    const int swz = lane & 7;
    float2 xp[C];
#pragma unroll
    for (int i = 0; i < C / 2; ++i) {
      const float4 v = *reinterpret_cast<const float4*>(slot + ((i ^ swz) << 2));
      xp[2 * i] = make_float2(v.x, v.y);
      xp[2 * i + 1] = make_float2(v.z, v.w);
    }
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j) {
      float2 a = acc[j];
      const BlockC12 A = decode_c12_v<V>(cur.r[j].x, cur.e[j], lane8, tabs);
      const BlockC12 B = decode_c12_v<V>(cur.r[j].y, cur.e[j] >> 4, lane8, tabs);
      const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
#if SEEDLM_GEMV_C12_ORDER == 1
      // Window-major: each of the 32 stream windows is formed once and feeds
      // the (up to two) states that sit in its halves.
      int32_t va[12], vb[12];
#pragma unroll
      for (int c = 0; c < 12; ++c) { va[c] = A.init; vb[c] = B.init; }
      c12_windows<0>(A, B, va, vb);
#pragma unroll
      for (int c = 0; c < 12; ++c) a = fma_pair(va[c], vb[c], negm, xp[c], a);
#else
#define SEEDLM_C12_STEP(c) a = fma_pair(weight_bits_c12<c>(A), weight_bits_c12<c>(B), negm, xp[c], a);
      SEEDLM_C12_STEP(0) SEEDLM_C12_STEP(1) SEEDLM_C12_STEP(2) SEEDLM_C12_STEP(3)
      SEEDLM_C12_STEP(4) SEEDLM_C12_STEP(5) SEEDLM_C12_STEP(6) SEEDLM_C12_STEP(7)
      SEEDLM_C12_STEP(8) SEEDLM_C12_STEP(9) SEEDLM_C12_STEP(10) SEEDLM_C12_STEP(11)
#undef SEEDLM_C12_STEP
#endif
      acc[j] = a;
    }
  }
}

// One launch may run several independent GEMVs of the same format (a
// batch): the tables are filled once, and each CTA then takes its share of
// every GEMV in turn.
constexpr int kMaxBatch = 8;
struct GemvBatch {
  int n;
  GemvGeom g[kMaxBatch];
  const uint32_t* rec[kMaxBatch];
  const uint8_t* ep[kMaxBatch];
  const uint16_t* x[kMaxBatch];
  float* y[kMaxBatch];
};

// For every GEMV of the batch, CTA b owns the contiguous row groups
// [g0, g1) (sizes differ by at most one group), processed in passes of at
// most pass_groups groups.  Within a pass, x is staged one column segment at
// a time (once per GEMV when one segment holds all of x); the (group, span)
// items of the pass and segment are split into equal contiguous ranges, one
// per warp.  A warp walks its range with record sets loaded
// Tune<C, V>::kPrefetch items ahead (across group boundaries), and whenever it
// leaves a group it reduces its 4 row sums with shuffles and adds them into
// its own slot of the pass's partial sums.  At the end of the pass the slots
// of each row are added in warp order and written.
template <int C, int V, bool kBatch>
__global__ void __launch_bounds__(Tune<C, V>::kWarps * 32, Tune<C, V>::kMinBlocks)
gemv_kernel(const __grid_constant__ GemvBatch B, int is_bf16) {
  constexpr int kP = Tune<C, V>::kPrefetch;
  constexpr int kSU = span_units<V>(), kRPI = rows_per_item<V>();
  extern __shared__ __align__(16) unsigned char smem[];
  // V = 0: the table addresses are absolute, so the allocation must start at
  // kSmemBase.
  if (V != 1 && smem_u32(smem) != kSmemBase) {
    if (threadIdx.x == 0) atomicOr(&g_gemv_error, 1u);
    return;
  }
  const unsigned char* tabs = smem;
  float* xs = reinterpret_cast<float*>(smem + Smem<C, V>::kXOff);
  float* part = reinterpret_cast<float*>(smem + Smem<C, V>::kPartOff);
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = Smem<C, V>::kXBytes / 4;
                    const int part_floats =
                        (int)(seedlm_dynamic_smem_bytes() - Smem<C, V>::kPartOff) / 4;)
  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lane4 = (uint32_t)lane << 2, lane8 = (uint32_t)(lane & 15) << 3;
  RecSet<C, V> buf[kP + 1];

  // The next kernel in the stream may launch now: its CTAs take an SM as
  // soon as this kernel's CTA there exits, and run their own prologue while
  // the slower CTAs of this grid finish.  Every CTA of this grid is resident
  // before the trigger completes, so the early start cannot starve it.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (C == 8 && (int64_t)B.g[0].rows * B.g[0].rec_pitch >= kL2PrefetchMinWords) {
    // The warp's first record sets of the first GEMV head for L2 while the
    // tables are filled and the previous kernel finishes: after the wait
    // they come from L2, not from DRAM.  Measured per launch: 0.4-1.7 us
    // faster on 8192 x 8192 and larger, 0.1-0.7 us slower on smaller
    // matrices (hence the size floor); at 3 bits (records and exponent
    // bytes) 0.2-1 us slower.
    const GemvGeom& g = B.g[0];
    const int g0 = (int)((int64_t)blockIdx.x * g.groups / gridDim.x);
    const int g1 = (int)((int64_t)(blockIdx.x + 1) * g.groups / gridDim.x);
    const int sl = min(g.seg_spans, g.n_spans);
    const int items = (min(g0 + g.pass_groups, g1) - g0) * sl;
    const int i0 = (int)((int64_t)warp * items / nw);
    const int i1 = (int)((int64_t)(warp + 1) * items / nw);
    int grp = g0 + (sl > 0 ? i0 / sl : 0), span = sl > 0 ? i0 % sl : 0;
    for (int k = 0; k < 2 * (kP + 1) && i0 + k < i1; ++k) {
      prefetch_set<C, V>(B.rec[0], g, grp, span, lane);
      if (++span == sl) { span = 0; ++grp; }
    }
  }
  fill_tables<C, V>(smem);
  // Records and x may be the previous kernel's output: read them only now.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int nbatch = kBatch ? B.n : 1;
  for (int bi = 0; bi < nbatch; ++bi) {
    // The geometry stays in the parameter space and is read where used: held
    // in registers across the loop it made the 4-bit batch kernel spill, and
    // every variant measured 0.3-0.8 us slower per launch.
    const GemvGeom& g = B.g[bi];
    // One GEMV keeps its pointers in registers; a batch reads them from the
    // parameter where used (each choice measured faster for its kind).
    const uint32_t* __restrict__ rec_r = kBatch ? nullptr : B.rec[0];
    const uint8_t* __restrict__ ep_r = kBatch ? nullptr : B.ep[0];
    const uint16_t* __restrict__ x_r = kBatch ? nullptr : B.x[0];
    float* __restrict__ y_r = kBatch ? nullptr : B.y[0];
#define SEEDLM_PTR(reg, field) (kBatch ? B.field[bi] : reg)
    const int g0 = (int)((int64_t)blockIdx.x * g.groups / gridDim.x);
    const int g1 = (int)((int64_t)(blockIdx.x + 1) * g.groups / gridDim.x);
    for (int p0 = g0; p0 < g1; p0 += g.pass_groups) {
      const int p1 = min(p0 + g.pass_groups, g1);
      // Partial sums of the pass: warp w's sum for row t at part[w * pass_rows + t],
      // so the final reduction reads consecutive words across the threads.
      const int pass_rows = (p1 - p0) * kRPI;
      for (int i = threadIdx.x; i < pass_rows * nw; i += blockDim.x)
        if (SEEDLM_IN_BOUNDS(g_check_flag, i, part_floats)) part[i] = 0.f;
      for (int sg = 0; sg < g.n_segs; ++sg) {
        const int s0 = sg * g.seg_spans;
        const int sl = min(g.seg_spans, g.n_spans - s0);
        const int items = (p1 - p0) * sl;
        const int i0 = (int)((int64_t)warp * items / nw);
        const int i1 = (int)((int64_t)(warp + 1) * items / nw);
        // Item cursor (grp, span) and load cursor (lgrp, lspan), kP items
        // ahead.  The first record sets do not depend on x: they are in
        // flight while x is staged.
        int grp = p0 + i0 / sl, span = i0 % sl;
        int lgrp = grp, lspan = span;
#pragma unroll
        for (int k = 0; k <= kP; ++k) {
          if (i0 + k < i1) load_set<C, V>(buf[k], SEEDLM_PTR(rec_r, rec), SEEDLM_PTR(ep_r, ep), g, lgrp, s0 + lspan, lane);
          if (++lspan == sl) { lspan = 0; ++lgrp; }
        }
        // One segment: x stays staged for every pass of this GEMV.
        if (g.n_segs > 1 || p0 == g0) stage_x<C, V>(xs, SEEDLM_PTR(x_r, x), is_bf16, g, s0, sl);
        __syncthreads();  // x, tables and zeroed partials ready
        if (i0 < i1) {
          float2 acc[kRowsPerTask];
#pragma unroll
          for (int j = 0; j < kRowsPerTask; ++j) acc[j] = make_float2(0.f, 0.f);
          int ci = i0;
          for (;;) {
#pragma unroll
            for (int k = 0; k <= kP; ++k) {
              const int ul = span * kSU + lane % kSU;
              // Every x slot of the lane's unit lies in its kSlotFloats row.
              if (SEEDLM_IN_BOUNDS(g_check_flag, (ul + 1) * (Smem<C, V>::kSlotFloats) - 1, xs_floats))
                rebuild_and_dot<C, V>(buf[k], xs, ul, lane, lane4, lane8, tabs, acc);
              if (ci + kP + 1 < i1) {
                load_set<C, V>(buf[k], SEEDLM_PTR(rec_r, rec), SEEDLM_PTR(ep_r, ep), g, lgrp, s0 + lspan, lane);
                if (++lspan == sl) { lspan = 0; ++lgrp; }
              }
              ++ci;
              const bool end_group = (++span == sl);
              if (end_group || ci == i1) {
#pragma unroll
                for (int j = 0; j < kRowsPerTask; ++j) {
                  // Sum over the lanes of the row's span (the warp, or its half).
                  float sum = acc[j].x + acc[j].y;
#pragma unroll
                  for (int o = kSU / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                  const int pi = warp * pass_rows + (grp - p0) * kRPI + (lane / kSU) * kRowsPerTask + j;
                  if (lane % kSU == 0 && SEEDLM_IN_BOUNDS(g_check_flag, pi, part_floats)) part[pi] += sum;
                  acc[j] = make_float2(0.f, 0.f);
                }
                if (end_group) { span = 0; ++grp; }
                if (ci == i1) goto range_done;
              }
            }
          }
        range_done:;
        }
        __syncthreads();  // partials complete; x may be restaged
      }
      for (int t = threadIdx.x; t < pass_rows; t += blockDim.x) {
        const int r = p0 * kRPI + t;
        if (r < g.rows) {
          float sum = 0.f;
          for (int w = 0; w < nw; ++w)
            if (SEEDLM_IN_BOUNDS(g_check_flag, w * pass_rows + t, part_floats)) sum += part[w * pass_rows + t];
          if (SEEDLM_IN_BOUNDS(g_check_flag, r, g.rows)) SEEDLM_PTR(y_r, y)[r] = sum;
        }
      }
      __syncthreads();  // partials read before the next pass clears them
    }
  }
}

#undef SEEDLM_PTR

template <int C, int V>
int warps_for(int items_per_cta) {
  int w = items_per_cta < Tune<C, V>::kWarps ? items_per_cta : Tune<C, V>::kWarps;
  // At least kMinWarps: on small matrices the CTA's setup (tables and x into
  // shared memory) outweighs its one or two items, and warps without items
  // still share it.
  return w < kMinWarps ? kMinWarps : w;
}

// Partial-sum bytes the small variant allows itself (keeps several CTAs per SM).
constexpr int kSmallPartBytes = 16384;

// The geometry for `nw` warps per CTA and `grid` CTAs, with the largest
// partial-sum pass that fits; pass_groups = 0 if even one group does not.
template <int C, int V>
GemvGeom make_geom(const seedlm_format& f, int max_smem, int nw, int grid) {
  constexpr int kBPL = Tune<C, V>::kBPL;
  GemvGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  constexpr int kSU = span_units<V>(), kRPI = rows_per_item<V>();
  g.n_spans = ((f.nb + kBPL - 1) / kBPL + kSU - 1) / kSU;
  if (g.n_spans < 1) g.n_spans = 1;
  g.groups = (f.rows + kRPI - 1) / kRPI;
  g.full_groups = f.rows / kRPI;
  // Units of the pitch: a span is full when its last unit ends inside it.
  g.full_spans = f.rec_pitch / (kBPL * kSU);
  g.n_segs = (g.n_spans + Smem<C, V>::kMaxSegSpans - 1) / Smem<C, V>::kMaxSegSpans;
  g.seg_spans = (g.n_spans + g.n_segs - 1) / g.n_segs;
  int64_t room = (int64_t)max_smem - Smem<C, V>::kPartOff;
  if (V == 1 && room > kSmallPartBytes) room = kSmallPartBytes;
  const int64_t per_group = (int64_t)Smem<C, V>::kPartBytesPerGroup * nw;
  const int max_cta_groups = grid > 0 ? (g.groups + grid - 1) / grid : 1;
  int64_t pg = room > 0 ? room / per_group : 0;
  if (pg > max_cta_groups) pg = max_cta_groups;
  g.pass_groups = (int)pg;
  return g;
}

template <int C, int V>
size_t smem_for(const GemvGeom& g, int nw) {
  return (size_t)Smem<C, V>::kPartOff + (size_t)g.pass_groups * Smem<C, V>::kPartBytesPerGroup * nw;
}

struct GemvLaunch {
  GemvBatch b;
  int grid, warps, variant;
  size_t smem;
};

// Work items (row group x span) of the busiest CTA, for a grid of up to
// max_ctas CTAs.
template <int C, int V>
int max_items_per_cta(const seedlm_format* const* f, int n, int max_ctas, int* max_groups) {
  constexpr int kBPL = Tune<C, V>::kBPL;
  int mi = 1;
  *max_groups = 1;
  constexpr int kSU = span_units<V>(), kRPI = rows_per_item<V>();
  for (int k = 0; k < n; ++k) {
    const int groups = (f[k]->rows + kRPI - 1) / kRPI;
    int n_spans = ((f[k]->nb + kBPL - 1) / kBPL + kSU - 1) / kSU;
    if (n_spans < 1) n_spans = 1;
    if (groups > *max_groups) *max_groups = groups;
    const int grid_k = groups < max_ctas ? groups : max_ctas;
    const int items = (groups + grid_k - 1) / (grid_k > 0 ? grid_k : 1) * n_spans;
    if (items > mi) mi = items;
  }
  return mi;
}

// One launch for n GEMVs of format C in variant V: one CTA per SM for V = 0
// (fewer if no GEMV has that many row groups), up to two per SM for V = 1;
// warps for the largest share, and each GEMV's partial-sum pass sized for
// that warp count.
template <int C, int V>
GemvLaunch plan_v(const seedlm_format* const* f, int n, const DeviceInfo& dev) {
  GemvLaunch L{};
  const int max_ctas = (V != 1) ? dev.num_sms : 2 * dev.num_sms;
  int max_groups = 1;
  const int max_items = max_items_per_cta<C, V>(f, n, max_ctas, &max_groups);
  L.variant = V;
  L.grid = max_groups < max_ctas ? max_groups : max_ctas;
  L.warps = warps_for<C, V>(max_items);
  L.b.n = n;
  L.smem = 0;
  for (int k = 0; k < n; ++k) {
    L.b.g[k] = make_geom<C, V>(*f[k], dev.max_smem_optin, L.warps, L.grid);
    if (L.b.g[k].pass_groups == 0) {
      L.smem = 0;
      return L;
    }
    const size_t sm = smem_for<C, V>(L.b.g[k], L.warps);
    if (sm > L.smem) L.smem = sm;
  }
  return L;
}

// The small variant when the large one would give each of its 16 warps
// fewer than 4 items: there the setup of the replicated tables and the
// one-CTA-per-SM launch, not the rebuild, set the time.
// Lane units the busiest of `grid` CTAs walks through in variant V (row
// groups per CTA rounded up, each row's units padded to whole spans), summed
// over the batch's products.
template <int V>
int64_t busiest_cta_units(const seedlm_format* const* f, int n, int bpl, int grid) {
  constexpr int kSU = span_units<V>(), kRPI = rows_per_item<V>();
  int64_t t = 0;
  for (int k = 0; k < n; ++k) {
    const int64_t units = (f[k]->nb + bpl - 1) / bpl;
    const int64_t groups = (f[k]->rows + kRPI - 1) / kRPI;
    t += (groups + grid - 1) / grid * kRPI * ((units + kSU - 1) / kSU * kSU);
  }
  return t;
}

template <int C>
GemvLaunch plan(const seedlm_format* const* f, int n, const DeviceInfo& dev) {
  int max_groups = 1;
  const int items = max_items_per_cta<C, 0>(f, n, dev.num_sms, &max_groups);
  if (items < 4 * Tune<C, 0>::kWarps) return plan_v<C, 1>(f, n, dev);
  if constexpr (C == 12) {
    // Half-warp spans where the busiest CTA then has less to do: less span
    // padding, against coarser row groups (8 rows) to spread over the CTAs.
    constexpr int kBPL = Tune<12, 0>::kBPL;
    if (busiest_cta_units<2>(f, n, kBPL, dev.num_sms) < busiest_cta_units<0>(f, n, kBPL, dev.num_sms))
      return plan_v<12, 2>(f, n, dev);
  }
  return plan_v<C, 0>(f, n, dev);
}

}  // namespace

size_t gemv_smem_bytes(const seedlm_format& f, const DeviceInfo& dev) {
  const seedlm_format* fp = &f;
  return f.C == 8 ? plan<8>(&fp, 1, dev).smem : plan<12>(&fp, 1, dev).smem;
}

int read_and_clear_gemv_error(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof(v));
  if (err != cudaSuccess) return record_cuda_error(err);
  if (v) {
    err = cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof(zero));
    if (err != cudaSuccess) return record_cuda_error(err);
  }
  *out = v;
  return SEEDLM_OK;
}

const void* kernel_for(int C, int V, bool batch) {
  if (C == 8) {
    if (V == 0) return batch ? (const void*)gemv_kernel<8, 0, true> : (const void*)gemv_kernel<8, 0, false>;
    return batch ? (const void*)gemv_kernel<8, 1, true> : (const void*)gemv_kernel<8, 1, false>;
  }
  if (V == 0) return batch ? (const void*)gemv_kernel<12, 0, true> : (const void*)gemv_kernel<12, 0, false>;
  if (V == 2) return batch ? (const void*)gemv_kernel<12, 2, true> : (const void*)gemv_kernel<12, 2, false>;
  return batch ? (const void*)gemv_kernel<12, 1, true> : (const void*)gemv_kernel<12, 1, false>;
}

int launch_gemv_batch(int n, const seedlm_format* const* f, const uint32_t* const* rec,
                      const uint8_t* const* eplane, const uint16_t* const* x, int is_bf16,
                      float* const* y, cudaStream_t stream, const DeviceInfo& dev) {
  if (n < 1) return SEEDLM_OK;
  if (n > kMaxBatch) return SEEDLM_EUNSUPPORTED;
  const int C = f[0]->C;
  GemvLaunch L = (C == 8) ? plan<8>(f, n, dev) : plan<12>(f, n, dev);
  if (L.smem == 0) return SEEDLM_EUNSUPPORTED;  // the tables do not fit
  for (int k = 0; k < n; ++k) {
    L.b.rec[k] = rec[k];
    L.b.ep[k] = eplane[k];
    L.b.x[k] = x[k];
    L.b.y[k] = y[k];
  }
  const bool batch = n > 1;
  const void* kern = kernel_for(C, L.variant, batch);
  int rc = allow_max_smem(kern, dev);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.grid);
  cfg.blockDim = dim3(L.warps * 32);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {(void*)&L.b, (void*)&is_bf16};
  cudaError_t err = cudaLaunchKernelExC(&cfg, kern, args);
  if (err != cudaSuccess) return record_cuda_error(err);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

int launch_gemv(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                const DeviceInfo& dev) {
  if (f.rows == 0) return SEEDLM_OK;
  if (gemv_amort_applies(f, dev)) return launch_gemv_amort(f, rec, eplane, x, is_bf16, y, stream, dev);
  const seedlm_format* fp = &f;
  return launch_gemv_batch(1, &fp, &rec, &eplane, &x, is_bf16, &y, stream, dev);
}

}  // namespace seedlm
