// gemm_tc.cu -- Y = X W^T for a small batch on the 5th-generation tensor
// cores (tcgen05), with W rebuilt on the fly.
//
// Where the batch makes the product a real contraction (several rows of X
// share every rebuilt weight), the reconstructed tiles feed tcgen05.mma
// (paperhub.cn review thread: the weights are rebuilt from s and t and then
// used to compute the activations).  The MMAs are kind::f16 (K = 16) in the
// activations' own type, with W split exactly into pieces of that type:
//
//   * bf16 X: W = p1 + p2 + p3, three bf16 pieces (8 significant bits each;
//     a rebuilt weight has at most 20);
//   * fp16 X: 2^6 W = p1 + p2, two fp16 pieces (11 significant bits each; the
//     2^6 keeps the smallest weight quantum, 2^-30, at or above fp16's 2^-24)
//     and Y is scaled back by 2^-6.
//
// Every product of a piece and an activation is exact in the fp32 accumulator.
// One call is two launches:
//
//   1. stage_x_kernel copies X (M x cols) into the workspace in the
//      tensor-core operand layout, one contiguous slab per K chunk (NB x KC
//      16-bit elements, NB = M rounded up to 16, zero-padded), so the GEMM
//      copies a chunk of X into shared memory with a single bulk copy.
//   2. gemm_tc_kernel, one CTA per SM.  The work is the list of
//      (128-row tile, K chunk) units in tile-major order, cut into equal
//      contiguous ranges, one per CTA ("stream-K"), so every SM gets the same
//      number of units whatever the shape.  Inside a CTA:
//        * 16 producer warps rebuild the unit's 128 x KC weights exactly in
//          fp32 (seedlm_device.cuh), split them into pieces, pack two K
//          neighbours per 32-bit word and store them straight into tensor
//          memory with tcgen05.st -- A operand stages, 128 lanes = rows.  Warp
//          w owns TMEM lanes 32(w%4).. and a quarter (w/4) of the chunk's
//          blocks.
//        * one thread issues the MMAs (M = 128, N = NB, A from TMEM, B = X
//          slab from shared memory), all pieces into the same fp32
//          accumulator in TMEM.  An MMA of this shape costs the tensor core
//          about 45 cycles whatever N (<= 64) and K (8 for tf32, 16 here), so
//          K = 16 halves the MMA count of a tf32 hi/lo split for fp16 X.
//        * one thread keeps the X slabs coming, a few chunks ahead, with bulk
//          copies.
//        * stages are handed over with mbarriers only (A stage full: all 16
//          producer warps arrived; A stage / X slab free: tcgen05.commit of the
//          MMAs that read it), so no warp waits for the whole CTA.
//        * the accumulator is double-buffered in TMEM.  At the end of each
//          tile segment warps 0-3 read it out: a tile owned by one CTA goes
//          straight to Y; otherwise each CTA writes a partial tile to the
//          workspace and the last of the tile's CTAs to arrive (atomic
//          counter) adds the partials in CTA order -- a fixed order, so every
//          call gives the same bits -- writes Y and resets the counter.
//   Every mbarrier wait is bounded; a wait that gives up raises the library's
//   device error flag, and TMEM is always released.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"
#include "tcgen05.cuh"

namespace seedlm {

__device__ unsigned int g_tc_error = 0;

SEEDLM_CHECK_FLAG(gemm_tc)

namespace {

constexpr int kTileM = 128;
constexpr int kProdWarps = 16;
constexpr int kMmaWarp = kProdWarps;         // issues the MMAs (one thread)
constexpr int kLoaderWarp = kProdWarps + 1;  // copies the X slabs (one thread)
constexpr int kThreads = (kProdWarps + 2) * 32;
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimit = 2000000000ull;  // ns an mbarrier wait may take before giving up

// Per format and piece count (PC = 3: bf16 pieces, PC = 2: fp16 pieces):
// K columns per unit, blocks per producer thread and unit, A stages in TMEM
// (PC x KC/2 columns each, two 16-bit elements per column), X slabs in
// shared memory.
template <int C, int PC>
struct TcCfg;
template <int PC>
struct TcCfg<8, PC> {
  static constexpr int KC = 128;  // 16 blocks
  static constexpr int BPT = 4;
  static constexpr int AS = (PC == 3) ? 2 : 3;
  static constexpr int XS = 5;
};
template <int PC>
struct TcCfg<12, PC> {
  static constexpr int KC = 96;  // 8 blocks
  static constexpr int BPT = 2;
  static constexpr int AS = (PC == 3) ? 2 : 3;
  static constexpr int XS = 5;
};
constexpr int kRecAhead = 2;   // units of records a producer thread has in flight

struct TcGeom {
  int rows, cols, nb, rec_pitch, e_pitch, M;
  int nchunks, tiles;
  long long units;  // tiles * nchunks
  int segs_max;     // most tiles any one CTA touches
};

template <int C, int NB, int PC>
struct TcSmem {
  static constexpr int KC = TcCfg<C, PC>::KC;
  static constexpr int AS = TcCfg<C, PC>::AS;
  static constexpr int XS = TcCfg<C, PC>::XS;
  static constexpr int BPT = TcCfg<C, PC>::BPT;
  static constexpr int SBO = KC * 16;  // bytes between 8-row groups of X (KC/8 core matrices)
  static constexpr int XB = NB * KC * 2;  // one X slab (16-bit elements)
  static constexpr int PIECE_COLS = KC / 2;      // TMEM columns of one piece of a stage
  static constexpr int STAGE_COLS = PC * PIECE_COLS;
  static constexpr int TABLE_OFF = XS * XB;
  // C = 8: jump tables (2 KB) + coefficient tables (4 KB); C = 12: jump tables.
  static constexpr int TABLE_BYTES = (C == 8) ? 512 * 4 + 512 * 8 : 512 * 8;
  static constexpr int BAR_OFF = TABLE_OFF + TABLE_BYTES;
  // mbarriers: xfull[XS] xfree[XS] afull[AS] afree[AS] dfree[2]
  static constexpr int NBAR = 2 * XS + 2 * AS + 2;
  static constexpr int SLOT_OFF = BAR_OFF + 8 * NBAR;  // TMEM base, last-CTA flag, give-up flag
  static constexpr int TOTAL = SLOT_OFF + 16;
  static constexpr int D_COL = AS * STAGE_COLS;  // first accumulator column
  static_assert(D_COL + 2 * 64 <= kTmemCols, "TMEM budget");
  static_assert(KC == 4 * BPT * C, "four producer quarters of BPT blocks per unit");
  static_assert(KC % 16 == 0, "whole K = 16 MMA steps");
};

// Byte offset of X element (n, k) inside a slab (K-major core matrices:
// 8 rows x 16 bytes = 8 elements, adjacent along K at 128 B, 8-row groups at
// SBO = KC * 16 bytes).
template <int KC>
__host__ __device__ constexpr int slab_byte(int n, int k) {
  return (n >> 3) * (KC * 16) + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2;
}

template <int KC, int NB>
__global__ void __launch_bounds__(256)
stage_x_kernel(const uint16_t* __restrict__ X, int M, int cols, int nchunks,
               unsigned char* __restrict__ Xs) {
  // The GEMM may start its prologue at once; it reads Xs only after
  // griddepcontrol.wait, i.e. after this grid has finished.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int PER_CHUNK = NB * (KC / 8);  // 16-byte groups per slab
  const long long total = (long long)nchunks * PER_CHUNK;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int chunk = (int)(i / PER_CHUNK);
    const int rem = (int)(i - (long long)chunk * PER_CHUNK);
    const int n = rem / (KC / 8), k8 = rem - n * (KC / 8);  // k fastest: coalesced reads
    const int col = chunk * KC + 8 * k8;
    uint32_t v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t a = (n < M && col + 2 * u < cols) ? X[(size_t)n * cols + col + 2 * u] : 0u;
      const uint32_t b = (n < M && col + 2 * u + 1 < cols) ? X[(size_t)n * cols + col + 2 * u + 1] : 0u;
      v[u] = a | (b << 16);
    }
    const size_t xb = (size_t)chunk * (NB * KC * 2) + slab_byte<KC>(n, 8 * k8);
    if (SEEDLM_IN_BOUNDS(g_check_flag, xb + 15, (size_t)nchunks * (NB * KC * 2)))
      *reinterpret_cast<uint4*>(Xs + xb) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

__device__ __forceinline__ long long unit_begin(int cta, long long units, int ctas) {
  return (long long)cta * units / ctas;
}
// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long u, long long units, int ctas) {
  return (int)(((u + 1) * ctas + units - 1) / units) - 1;
}

// Pieces of two rebuilt weights (K neighbours) given as magic-biased floats
// b (weight = b + nm), packed two per 32-bit word, the lower K index in the
// low half.  All splits are exact.
template <int PC>
__device__ __forceinline__ void split_pair(float b0, float b1, float nm, uint32_t (&out)[PC]) {
  if constexpr (PC == 3) {
    // bf16: each piece keeps the top 8 significant bits of what is left.
    const float2 w = __fadd2_rn(make_float2(b0, b1), make_float2(nm, nm));
    const uint32_t h0 = __float_as_uint(w.x) & 0xFFFF0000u, h1 = __float_as_uint(w.y) & 0xFFFF0000u;
    const float2 r = __ffma2_rn(make_float2(__uint_as_float(h0), __uint_as_float(h1)),
                                make_float2(-1.f, -1.f), w);
    const uint32_t m0 = __float_as_uint(r.x) & 0xFFFF0000u, m1 = __float_as_uint(r.y) & 0xFFFF0000u;
    const float2 l = __ffma2_rn(make_float2(__uint_as_float(m0), __uint_as_float(m1)),
                                make_float2(-1.f, -1.f), r);
    out[0] = prmt<0x7632u>(h0, h1);
    out[1] = prmt<0x7632u>(m0, m1);
    out[2] = prmt<0x7632u>(__float_as_uint(l.x), __float_as_uint(l.y));
  } else {
    // fp16 of 2^6 w: the top 11 significant bits, then the rest.
    const float2 w = __ffma2_rn(make_float2(b0, b1), make_float2(64.f, 64.f),
                                make_float2(64.f * nm, 64.f * nm));
    const uint32_t h0 = __float_as_uint(w.x) & 0xFFFFE000u, h1 = __float_as_uint(w.y) & 0xFFFFE000u;
    const float2 l = __ffma2_rn(make_float2(__uint_as_float(h0), __uint_as_float(h1)),
                                make_float2(-1.f, -1.f), w);
    const __half2 ph = __floats2half2_rn(__uint_as_float(h0), __uint_as_float(h1));
    const __half2 pl = __floats2half2_rn(l.x, l.y);
    out[0] = *reinterpret_cast<const uint32_t*>(&ph);
    out[1] = *reinterpret_cast<const uint32_t*>(&pl);
  }
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

template <int C, int NB, int PC>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
               const unsigned char* __restrict__ Xs, float* __restrict__ Y,
               float* __restrict__ partial, unsigned int* __restrict__ counters, TcGeom g) {
  using L = TcSmem<C, NB, PC>;
  constexpr int KC = L::KC, AS = L::AS, XS = L::XS, BPT = L::BPT;
  constexpr float kYScale = (PC == 2) ? 1.0f / 64.0f : 1.0f;  // undo the fp16 pieces' 2^6
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ctas = gridDim.x;
  // The whole shared-memory layout lies inside the launch's allocation
  // (checked before any barrier or TMEM exists, so leaving is safe).
  if (!SEEDLM_IN_BOUNDS(g_check_flag, L::TOTAL - 1, seedlm_dynamic_smem_bytes())) return;
  const long long u_begin = unit_begin(blockIdx.x, g.units, ctas);
  const int n_units = (int)(unit_begin(blockIdx.x + 1, g.units, ctas) - u_begin);
  const int t_first = (int)(u_begin / g.nchunks);
  const UnitCursor c0{t_first, (int)(u_begin - (long long)t_first * g.nchunks)};

  uint32_t* t32 = reinterpret_cast<uint32_t*>(smem + L::TABLE_OFF);
  uint2* t64 = reinterpret_cast<uint2*>(smem + L::TABLE_OFF);
  for (int i = tid; i < 512; i += kThreads) {
    uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
    if constexpr (C == 8)
      t32[i] = (uint32_t)v;
    else
      t64[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
  }
  if constexpr (C == 8) {
    uint2* tq = reinterpret_cast<uint2*>(t32 + 512);
    fill_coef_tables_c8(tq, tq + 256, tid, kThreads);
  }
  const uint32_t bar = tc::smem_u32(smem + L::BAR_OFF);
  // xfull: X slab landed.  xfree: the MMAs that read the slab completed.
  // afull: all producer warps stored the A stage.  afree: the unit's MMAs
  // completed: its A stage may be reused and, at a segment's end, the
  // accumulator is final.  dfree: warps 0-3 have read an accumulator out.
  auto xfull = [&](int s) { return bar + 8 * s; };
  auto xfree = [&](int s) { return bar + 8 * (XS + s); };
  auto afull = [&](int s) { return bar + 8 * (2 * XS + s); };
  auto afree = [&](int s) { return bar + 8 * (2 * XS + AS + s); };
  auto dfree = [&](int b) { return bar + 8 * (2 * XS + 2 * AS + b); };
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::SLOT_OFF);
  if (tid == 0) {
    for (int s = 0; s < XS; ++s) {
      tc::mbar_init(xfull(s), 1);
      tc::mbar_init(xfree(s), 1);
    }
    for (int s = 0; s < AS; ++s) {
      tc::mbar_init(afull(s), kProdWarps);
      tc::mbar_init(afree(s), 1);
    }
    for (int b = 0; b < 2; ++b) tc::mbar_init(dfree(b), 4);
    tc::fence_mbar_init();
    slot[2] = 0u;  // give-up flag shared by all bounded waits
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(slot), kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = slot[0];
  volatile uint32_t* abort_flag = slot + 2;
  bool ok = true;

  if (warp == kLoaderWarp) {
    // ------------------------------------------------ X slabs
    if (lane == 0) {
      const uint32_t xs0 = tc::smem_u32(smem);
      UnitCursor xc = c0;
      // Xs is written by the previous kernel on the stream.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int j = 0; j < n_units; ++j, xc.next(g.nchunks)) {
        const int s = j % XS;
        if (j >= XS)  // the slab's previous unit (j - XS) has finished its MMAs
          ok = tc::mbar_wait_or_abort(xfree(s), ((j / XS) - 1) & 1, kWaitLimit, abort_flag) && ok;
        if (SEEDLM_IN_BOUNDS(g_check_flag, xc.chunk, g.nchunks)) {
          tc::mbar_arrive_expect_tx(xfull(s), L::XB);
          tc::bulk_g2s(xs0 + s * L::XB, Xs + (size_t)xc.chunk * L::XB, L::XB, xfull(s));
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
      const uint32_t idesc = tc::idesc_f16(NB, PC == 3 ? 1 : 0);
      const uint64_t bdesc0 = tc::smem_desc(tc::smem_u32(smem), 128, L::SBO);  // slab 0, K slice 0
      int seg = 0;
      UnitCursor mc = c0;
      for (int i = 0; i < n_units; ++i, mc.next(g.nchunks)) {
        const bool first = i == 0 || mc.chunk == 0;
        if (first && i > 0) ++seg;
        const int db = seg & 1;
        if (first && seg >= 2)  // accumulator db was last used by segment seg - 2
          ok = tc::mbar_wait_or_abort(dfree(db), ((seg >> 1) - 1) & 1, kWaitLimit, abort_flag) && ok;
        const int xs = i % XS, as = i % AS;
        if (!tc::mbar_try_wait2(xfull(xs), (i / XS) & 1, afull(as), (i / AS) & 1)) {
          ok = tc::mbar_wait_or_abort(xfull(xs), (i / XS) & 1, kWaitLimit, abort_flag) && ok;
          ok = tc::mbar_wait_or_abort(afull(as), (i / AS) & 1, kWaitLimit, abort_flag) && ok;
        }
        __syncwarp();  // reconverge before the elected issue
        tc::fence_after_sync();
        // The issue rate bounds the kernel (an MMA of this shape takes the
        // tensor core about 45 cycles), so everything but the MMAs is
        // computed up front.
        const uint32_t a0 = tmem + as * L::STAGE_COLS;
        const uint32_t d = tmem + L::D_COL + 64 * db;
        const uint64_t bd = bdesc0 + (uint64_t)((xs * L::XB) >> 4);
        const uint32_t acc0 = first ? 0u : 1u;
#pragma unroll
        for (int kk = 0; kk < KC / 16; ++kk)
#pragma unroll
          for (int pc = 0; pc < PC; ++pc)
            tc::mma_f16_ts_warp(d, a0 + pc * L::PIECE_COLS + 8 * kk, bd + 16 * kk, idesc,
                                (kk == 0 && pc == 0) ? acc0 : 1u);
        tc::mma_commit_warp(afree(as));  // A stage free; at a segment's end the accumulator is final
        tc::mma_commit_warp(xfree(xs));  // X slab free
      }
      // The CTA releases TMEM only after its last MMAs have completed
      // (bounded, not cut short by the give-up flag).
      if (n_units > 0) {
        const int last = n_units - 1;
        ok = tc::mbar_wait(afree(last % AS), (last / AS) & 1, kWaitLimit) && ok;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ producers (+ epilogue)
    const int lq = warp & 3, kq = warp >> 2;
    const int prow = 32 * lq + lane;  // TMEM lane = row in the tile
    auto load_rec = [&](const UnitCursor& u, RecUnit<C>& p) {
      const int gr = u.tile * kTileM + prow;
      const int b0 = u.chunk * (KC / C) + kq * BPT;  // a multiple of BPT
      // The thread's last record and its exponent byte lie inside row gr.
      const bool ok_ = gr < g.rows && b0 < g.nb &&
                       SEEDLM_IN_BOUNDS(g_check_flag, b0 + BPT - 1, g.rec_pitch) &&
                       (C == 8 || SEEDLM_IN_BOUNDS(g_check_flag, b0 >> 1, g.e_pitch));
      const uint32_t* src = rec + (size_t)gr * g.rec_pitch + b0;
      if constexpr (C == 8) {
        const uint4 v = ok_ ? ld_stream_u4(src) : make_uint4(0u, 0u, 0u, 0u);
        p.r[0] = v.x; p.r[1] = v.y; p.r[2] = v.z; p.r[3] = v.w;
        p.e = 0;
      } else {
        const uint2 v = ok_ ? ld_stream_u2(src) : make_uint2(0u, 0u);
        p.r[0] = v.x; p.r[1] = v.y;
        p.e = ok_ ? (uint32_t)ld_stream_u8(eplane + (size_t)gr * g.e_pitch + (b0 >> 1)) : 0u;
      }
    };

    auto produce = [&](int i, const RecUnit<C>& cur) {
      const int as = i % AS;
      if (i >= AS) ok = tc::mbar_wait_or_abort(afree(as), ((i / AS) - 1) & 1, kWaitLimit, abort_flag) && ok;
      tc::fence_after_sync();
      // Piece pc of this thread's BPT * C weights: BPT * C / 2 packed columns.
      constexpr int NPACK = BPT * C / 2;
      const uint32_t col0 = tmem + ((uint32_t)(32 * lq) << 16) + as * L::STAGE_COLS + kq * NPACK;
      uint32_t pk[PC][NPACK];
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        float b[C];
        float nm;
        if constexpr (C == 8) {
          // With bf16 pieces (the busier integer pipe) the coefficient words
          // come from the shared tables, measured 2 % faster; with fp16
          // pieces computing them is 2 % faster.
          const uint2* tq1 = reinterpret_cast<const uint2*>(t32 + 512);
          const BlockC8 blk = (PC == 3) ? decode_c8_tab(cur.r[j], t32, t32 + 256, tq1, tq1 + 256)
                                        : decode_c8(cur.r[j], t32, t32 + 256);
          nm = __uint_as_float(blk.negm);
          b[0] = __int_as_float(weight_bits_c8<0>(blk));
          b[1] = __int_as_float(weight_bits_c8<1>(blk));
          b[2] = __int_as_float(weight_bits_c8<2>(blk));
          b[3] = __int_as_float(weight_bits_c8<3>(blk));
          b[4] = __int_as_float(weight_bits_c8<4>(blk));
          b[5] = __int_as_float(weight_bits_c8<5>(blk));
          b[6] = __int_as_float(weight_bits_c8<6>(blk));
          b[7] = __int_as_float(weight_bits_c8<7>(blk));
        } else {
          const BlockC12 blk = decode_c12(cur.r[j], (j ? cur.e >> 4 : cur.e) & 15u, t64, t64 + 256);
          nm = __uint_as_float(blk.negm);
          b[0] = __int_as_float(weight_bits_c12<0>(blk));
          b[1] = __int_as_float(weight_bits_c12<1>(blk));
          b[2] = __int_as_float(weight_bits_c12<2>(blk));
          b[3] = __int_as_float(weight_bits_c12<3>(blk));
          b[4] = __int_as_float(weight_bits_c12<4>(blk));
          b[5] = __int_as_float(weight_bits_c12<5>(blk));
          b[6] = __int_as_float(weight_bits_c12<6>(blk));
          b[7] = __int_as_float(weight_bits_c12<7>(blk));
          b[8] = __int_as_float(weight_bits_c12<8>(blk));
          b[9] = __int_as_float(weight_bits_c12<9>(blk));
          b[10] = __int_as_float(weight_bits_c12<10>(blk));
          b[11] = __int_as_float(weight_bits_c12<11>(blk));
        }
#pragma unroll
        for (int c = 0; c < C; c += 2) {
          uint32_t o[PC];
          split_pair<PC>(b[c], b[c + 1], nm, o);
#pragma unroll
          for (int pc = 0; pc < PC; ++pc) pk[pc][(j * C + c) / 2] = o[pc];
        }
      }
#pragma unroll
      for (int pc = 0; pc < PC; ++pc) {
        if constexpr (C == 8) {
          tc::tmem_st16(col0 + pc * L::PIECE_COLS, pk[pc]);
        } else {
#pragma unroll
          for (int q = 0; q < NPACK / 4; ++q) tc::tmem_st4(col0 + pc * L::PIECE_COLS + 4 * q, pk[pc] + 4 * q);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(afull(as));
    };

    // Warps 0-3 (all 128 TMEM lanes) drain the accumulator of a segment, 16
    // columns at a time.
    auto epilogue = [&](int seg, int tile, int i_last) {
      const int db = seg & 1;
      ok = tc::mbar_wait_or_abort(afree(i_last % AS), (i_last / AS) & 1, kWaitLimit, abort_flag) &&
           ok;
      tc::fence_after_sync();
      const int row = 32 * warp + lane;
      const int gr = tile * kTileM + row;
      const int first = unit_owner((long long)tile * g.nchunks, g.units, ctas);
      const int last = unit_owner((long long)(tile + 1) * g.nchunks - 1, g.units, ctas);
      float* mine = partial + ((size_t)blockIdx.x * g.segs_max + seg) * (NB * kTileM);
      // Extents: Y holds M x rows floats; the partial tiles ctas x segs_max
      // tiles of NB x 128 floats (one per segment of each CTA).
      SEEDLM_CHECK_ONLY(const size_t y_n = (size_t)g.M * g.rows;
                        const size_t part_n = (size_t)ctas * g.segs_max * (NB * kTileM);
                        const size_t mine_off = ((size_t)blockIdx.x * g.segs_max + seg) * (NB * kTileM);)
#pragma unroll
      for (int n16 = 0; n16 < NB / 16; ++n16) {
        float v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + L::D_COL + 64 * db + 16 * n16, v);
        if (first == last) {
          if (gr < g.rows) {
#pragma unroll
            for (int q = 0; q < 16; ++q)
              if (16 * n16 + q < g.M &&
                  SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(16 * n16 + q) * g.rows + gr, y_n))
                Y[(size_t)(16 * n16 + q) * g.rows + gr] = v[q] * kYScale;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q)
            if (SEEDLM_IN_BOUNDS(g_check_flag, seg, g.segs_max) &&
                SEEDLM_IN_BOUNDS(g_check_flag, mine_off + (16 * n16 + q) * kTileM + row, part_n))
              mine[(16 * n16 + q) * kTileM + row] = v[q] * kYScale;
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(dfree(db));
      if (first == last) return;
      __threadfence();
      tc::named_sync(128);
      if (tid == 0)
        slot[1] = SEEDLM_IN_BOUNDS(g_check_flag, tile, g.tiles) &&
                          atomicAdd(&counters[tile], 1u) == (unsigned)(last - first)
                      ? 1u
                      : 0u;
      tc::named_sync(128);
      if (slot[1]) {
        __threadfence();
        if (gr < g.rows) {
          // Y = partial(first) + partial(first + 1) + ... in CTA order.
          for (int c = first; c <= last; ++c) {
            const int cseg = tile - (int)(unit_begin(c, g.units, ctas) / g.nchunks);
            const float* p = partial + ((size_t)c * g.segs_max + cseg) * (NB * kTileM) + row;
            if (!SEEDLM_IN_BOUNDS(g_check_flag, cseg, g.segs_max) ||
                !SEEDLM_IN_BOUNDS(g_check_flag,
                                  ((size_t)c * g.segs_max + cseg) * (NB * kTileM) +
                                      (size_t)(g.M - 1) * kTileM + row,
                                  part_n))
              continue;
            for (int n = 0; n < g.M; ++n) {
              float* y = Y + (size_t)n * g.rows + gr;
              *y = (c == first) ? p[n * kTileM] : *y + p[n * kTileM];
            }
          }
        }
        if (tid == 0) counters[tile] = 0u;
      }
      tc::named_sync(128);  // slot[1] is rewritten by the next segment
    };

    RecUnit<C> ring[kRecAhead];
    UnitCursor rc = c0;  // next unit whose records are loaded
#pragma unroll
    for (int k = 0; k < kRecAhead; ++k)
      if (k < n_units) {
        load_rec(rc, ring[k]);
        rc.next(g.nchunks);
      }
    UnitCursor pc = c0;  // unit being rebuilt
    int seg = 0;
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
          if (i > 0 && pc.chunk == 0) ++seg;
          produce(i, cur);
          if (warp < 4 && (i == n_units - 1 || pc.chunk == g.nchunks - 1))
            epilogue(seg, pc.tile, i);
          pc.next(g.nchunks);
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

// K columns per unit (the same for both piece types).
int kc_of(int C) { return C == 8 ? TcCfg<8, 3>::KC : TcCfg<12, 3>::KC; }

TcGeom make_tc_geom(const seedlm_format& f, int M, const DeviceInfo& dev, int* ctas) {
  TcGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.M = M;
  const int KC = kc_of(f.C);
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

// Workspace: [tile counters][X slabs][partial tiles], each part 256-aligned.
struct TcWorkspace {
  int64_t cnt_bytes, xs_bytes, part_bytes;
  int64_t total() const { return cnt_bytes + xs_bytes + part_bytes; }
};

int64_t round256(int64_t v) { return (v + 255) / 256 * 256; }

TcWorkspace tc_workspace(const TcGeom& g, int C, int ctas) {
  const int NB = (g.M + 15) / 16 * 16;
  TcWorkspace w;
  w.cnt_bytes = round256((int64_t)g.tiles * 4);
  w.xs_bytes = round256((int64_t)g.nchunks * NB * kc_of(C) * 2);
  w.part_bytes = round256((int64_t)ctas * g.segs_max * NB * kTileM * 4);
  return w;
}

template <int C, int NB, int PC>
int launch_tc(const TcGeom& g, int ctas, const uint32_t* rec, const uint8_t* eplane,
              const uint16_t* X, float* Y, unsigned char* ws, const TcWorkspace& w,
              cudaStream_t stream, const DeviceInfo& dev) {
  using L = TcSmem<C, NB, PC>;
  if ((size_t)L::TOTAL > (size_t)dev.max_smem_optin) return SEEDLM_EUNSUPPORTED;
  int rc = allow_max_smem((const void*)gemm_tc_kernel<C, NB, PC>, dev);
  if (rc) return rc;
  unsigned int* counters = reinterpret_cast<unsigned int*>(ws);
  unsigned char* xs = ws + w.cnt_bytes;
  float* partial = reinterpret_cast<float*>(ws + w.cnt_bytes + w.xs_bytes);

  const long long groups = (long long)g.nchunks * NB * (L::KC / 8);
  long long want = (groups + 255) / 256;
  const long long cap = 8ll * dev.num_sms;
  const int sgrid = (int)(want < cap ? (want < 1 ? 1 : want) : cap);
  stage_x_kernel<L::KC, NB><<<sgrid, 256, 0, stream>>>(X, g.M, g.cols, g.nchunks, xs);
  count_launch();
  if ((rc = record_cuda_error(cudaGetLastError()))) return rc;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::TOTAL;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<C, NB, PC>, rec, eplane,
                                       (const unsigned char*)xs, Y, partial, counters, g);
  if (err != cudaSuccess) return record_cuda_error(err);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

template <int C, int PC>
int dispatch_nb(const TcGeom& g, int ctas, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* X, float* Y, unsigned char* ws, const TcWorkspace& w,
                cudaStream_t st, const DeviceInfo& dev) {
  switch ((g.M + 15) / 16 * 16) {
    case 16: return launch_tc<C, 16, PC>(g, ctas, rec, eplane, X, Y, ws, w, st, dev);
    case 32: return launch_tc<C, 32, PC>(g, ctas, rec, eplane, X, Y, ws, w, st, dev);
    case 48: return launch_tc<C, 48, PC>(g, ctas, rec, eplane, X, Y, ws, w, st, dev);
    default: return launch_tc<C, 64, PC>(g, ctas, rec, eplane, X, Y, ws, w, st, dev);
  }
}

// bf16 activations take three bf16 pieces of W, fp16 activations two fp16
// pieces (of 2^6 W): A and B of one MMA always have the same type.
int dispatch_tc(const seedlm_format& f, const TcGeom& g, int ctas, const uint32_t* rec,
                const uint8_t* eplane, const uint16_t* X, int is_bf16, float* Y,
                unsigned char* ws, const TcWorkspace& w, cudaStream_t st, const DeviceInfo& dev) {
  if (f.C == 8)
    return is_bf16 ? dispatch_nb<8, 3>(g, ctas, rec, eplane, X, Y, ws, w, st, dev)
                   : dispatch_nb<8, 2>(g, ctas, rec, eplane, X, Y, ws, w, st, dev);
  return is_bf16 ? dispatch_nb<12, 3>(g, ctas, rec, eplane, X, Y, ws, w, st, dev)
                 : dispatch_nb<12, 2>(g, ctas, rec, eplane, X, Y, ws, w, st, dev);
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
