// gemm_cc.cu -- Y = X W^T for 2 to 4 rows of X and 3-bit blocks (C = 12,
// P = 4) on the CUDA cores, with W rebuilt block by block on the fly.
//
// SeedLM inference rebuilds each block from its seed and coefficients and
// multiplies it with the activations at once (paperhub.cn review thread,
// authors' reply on how inference uses s and t).  With a few activation rows
// the rebuild, not the multiply, is the work.  A 3-bit block is expensive to
// rebuild (four dp2a per weight, its 48 states twelve bits apart): the
// tensor-core kernel (gemm_tc.cu) adds an exact split of every weight into
// fp16 pieces and the hand-over to the MMA, and took as long at M = 2 as at
// M = 16.  Here every rebuilt weight pair feeds MB packed fp32 FMAs, one per
// row of X, the GEMV's design (gemv.cu) widened from one x to MB:
//
//   * lane-replicated decode tables at fixed shared addresses
//     (rep_tables.cuh), one CTA of 16 warps per SM, filled before
//     griddepcontrol.wait; records and X are read only after it;
//   * X staged as fp32 in shared memory, one column segment at a time: the
//     slot of lane unit u (one block, C columns) holds, for each weight pair
//     p and row m of X, the float2 (x_m[2p], x_m[2p+1]); its float4s are
//     XOR-swizzled by u so the 8 lanes of a quarter-warp hit distinct banks;
//   * an item is R rows of W x one span of 32 blocks (one per lane; R = 4,
//     or 2 with 4 rows of X): the lane loads its R records (one 4-byte load
//     per row, coalesced across the warp) an item ahead, takes its slot's x
//     values into registers once for the R rows, and per weight pair issues
//     one packed add (int -> float) and MB packed FMAs; acc[r][m] holds the
//     pair's two partial sums;
//   * a CTA owns a contiguous range of R-row groups, walked in passes that
//     fit the partial sums; within a pass and segment the (group, span)
//     items are split into equal contiguous ranges, one per warp.  When a
//     warp leaves a group it reduces its sums with shuffles into its own
//     shared-memory slots; at the end of the pass the slots are added in
//     warp order (the same order on every call) and Y is written.
//
// The sums are fp32 over exact weights and exact fp32 activations, as in the
// GEMV, so the product meets the same 1e-5 * sum |w x| bound.  (4-bit blocks
// stay on the tensor cores: their rebuild is three times cheaper, so this
// kernel's per-item costs and the x segments -- a 4-bit span of x fills its
// shared memory three times faster -- left it no faster than gemm_tc.cu.)
#include <cuda_runtime.h>

#include "rep_tables.cuh"
#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

SEEDLM_CHECK_FLAG(gemm_cc)

namespace {

__device__ unsigned int g_cc_error = 0;

constexpr int kWarps = 16;
constexpr int kSpan = 32;  // lane units (blocks) per span

// Rows of W per item: 4, or 2 with 4 rows of X, whose 24 x pairs and 16
// sums would not leave registers for 4 rows.
template <int C, int MB>
__host__ __device__ constexpr int rows_per_item() { return MB > 2 ? 2 : 4; }

using rep::kSmemBase;

// Shared memory, by absolute address (the dynamic allocation starts at
// kSmemBase; checked at entry):
//   [kSmemBase, tables)   X slots of one column segment
//   [tables, 0x30000)     lane-replicated decode tables
//   [0x30000, ...)        partial sums of one pass
template <int C, int MB>
struct CcSmem {
  static constexpr int kEntries = C / 2 * MB;  // float2 entries (pair p, row m) per unit
  static constexpr int kUsedF4 = kEntries / 2;
  static constexpr int kSlotF4 = kUsedF4 <= 8 ? 8 : 16;  // the swizzle needs >= 8
  static constexpr int kSlotFloats = 4 * kSlotF4;
  static constexpr int kXBytes = (int)(rep::tables_begin<C>() - kSmemBase);
  static constexpr int kMaxSegSpans = kXBytes / (kSlotFloats * 4) / kSpan;
  static constexpr int kPartOff = (int)(rep::kEnd - kSmemBase);
  static constexpr int kRows = rows_per_item<C, MB>();
  static constexpr int kAhead = 1;  // items of records in flight ahead of the one rebuilt
  static_assert(C == 12, "3-bit blocks (C = 12, P = 4)");
  static constexpr int kPartBytesPerGroup = kRows * MB * kWarps * 4;
  static_assert(kEntries % 2 == 0 && kUsedF4 <= kSlotF4, "slot");
  static_assert(kMaxSegSpans >= 1, "one span of x fits");
};

struct CcGeom {
  int rows, cols, nb, rec_pitch, e_pitch, M;
  int groups;       // ceil(rows / rows per item)
  int n_spans;      // ceil(nb / 32)
  int seg_spans;    // spans per x segment (the last one may be shorter)
  int n_segs;
  int pass_groups;  // row groups per partial-sum pass
};

// Float index of entry e (pair e / MB, row e % MB) of unit u's slot.
template <int C, int MB>
__device__ __forceinline__ int slot_index(int u, int e) {
  using S = CcSmem<C, MB>;
  return u * S::kSlotFloats + (((e >> 1) ^ (u & 7)) << 2) + ((e & 1) << 1);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// X columns of spans [s0, s0 + sl), zero past cols and past M rows, into the
// segment's slots.  One thread per (unit, row of X).
template <int C, int MB>
__device__ void stage_x(float* xs, const uint16_t* __restrict__ X, int is_bf16, const CcGeom& g,
                        int s0, int sl, int vec) {
  const int units = sl * kSpan;
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = CcSmem<C, MB>::kXBytes / 4;)
  for (int i = threadIdx.x; i < units * MB; i += blockDim.x) {
    const int u = i / MB, m = i - u * MB;
    const int col0 = (s0 * kSpan + u) * C;
    const uint16_t* xr = X + (size_t)m * g.cols;
    uint16_t v[C];
    if (vec && m < g.M && col0 + C <= g.cols) {
      // col0 is a multiple of 4 columns: three 8-byte loads.
      const uint2* q2 = reinterpret_cast<const uint2*>(xr + col0);
#pragma unroll
      for (int k = 0; k < C / 4; ++k) {
        const uint2 q = q2[k];
        v[4 * k] = (uint16_t)q.x;
        v[4 * k + 1] = (uint16_t)(q.x >> 16);
        v[4 * k + 2] = (uint16_t)q.y;
        v[4 * k + 3] = (uint16_t)(q.y >> 16);
      }
    } else {
#pragma unroll
      for (int k = 0; k < C; ++k) v[k] = (m < g.M && col0 + k < g.cols) ? xr[col0 + k] : (uint16_t)0;
    }
#pragma unroll
    for (int p = 0; p < C / 2; ++p) {
      const int si = slot_index<C, MB>(u, p * MB + m);
      if (SEEDLM_IN_BOUNDS(g_check_flag, si + 1, xs_floats))
        *reinterpret_cast<float2*>(xs + si) =
            make_float2(act_to_float(v[2 * p], is_bf16), act_to_float(v[2 * p + 1], is_bf16));
    }
  }
}

// The records of one item for this lane: block u of each of the group's R
// rows (zero past `rows` and past the row pitch: their x is zero) and the
// exponent bytes holding block u's nibble.
template <int R>
struct CcRecs {
  uint32_t r[R];
  uint32_t e[R];
};

template <int C, int R>
__device__ __forceinline__ void load_recs(CcRecs<R>& o, const uint32_t* __restrict__ rec,
                                          const uint8_t* __restrict__ eplane, const CcGeom& g,
                                          int grp, int u) {
  const int row0 = grp * R;
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const int r = row0 + j;
    const bool ok = r < g.rows && u < g.rec_pitch &&
                    SEEDLM_IN_BOUNDS(g_check_flag, (size_t)r * g.rec_pitch + u,
                                     (size_t)g.rows * g.rec_pitch);
    o.r[j] = ok ? ld_stream_u1(rec + (size_t)r * g.rec_pitch + u) : 0u;
    const bool eok = r < g.rows && (u >> 1) < g.e_pitch &&
                     SEEDLM_IN_BOUNDS(g_check_flag, (size_t)r * g.e_pitch + (u >> 1),
                                      (size_t)g.rows * g.e_pitch);
    o.e[j] = eok ? (uint32_t)ld_stream_u8(eplane + (size_t)r * g.e_pitch + (u >> 1)) : 0u;
  }
}

// acc[j][m] += (rebuilt weights of block `rec` of row j) . (x_m of the block),
// two partial sums per float2 (even and odd weights).
template <int C, int MB, int R>
__device__ __forceinline__ void rebuild_and_dot(const CcRecs<R>& cur, const float2 (&xe)[C / 2 * MB],
                                                int u, uint32_t lane8, float2 (&acc)[R][MB]) {
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const uint32_t e4 = (cur.e[j] >> (4 * (u & 1))) & 15u;
    const BlockC12 b = rep::decode_c12_rep<0>(cur.r[j], e4, lane8);
    const float2 nm = make_float2(__uint_as_float(b.negm), __uint_as_float(b.negm));
#define SEEDLM_CC12_PAIR(p)                                                                    \
  {                                                                                            \
    const float2 w = __fadd2_rn(make_float2(__int_as_float(weight_bits_c12<2 * (p)>(b)),      \
                                            __int_as_float(weight_bits_c12<2 * (p) + 1>(b))), \
                                nm);                                                           \
    _Pragma("unroll") for (int m = 0; m < MB; ++m) acc[j][m] = __ffma2_rn(w, xe[(p) * MB + m], acc[j][m]); \
  }
    SEEDLM_CC12_PAIR(0) SEEDLM_CC12_PAIR(1) SEEDLM_CC12_PAIR(2)
    SEEDLM_CC12_PAIR(3) SEEDLM_CC12_PAIR(4) SEEDLM_CC12_PAIR(5)
#undef SEEDLM_CC12_PAIR
  }
}

template <int C, int MB>
__global__ void __launch_bounds__(kWarps * 32, 1)
gemm_cc_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
               const uint16_t* __restrict__ X, int is_bf16, int vec, float* __restrict__ Y,
               const __grid_constant__ CcGeom g) {
  using S = CcSmem<C, MB>;
  constexpr int kE = S::kEntries;
  constexpr int kRows = S::kRows;
  constexpr int kAhead = S::kAhead;
  extern __shared__ __align__(16) unsigned char smem[];
  // The next kernel in the stream may launch now (its CTAs take an SM when
  // this kernel's CTA there exits); every CTA of this grid is resident
  // before the trigger completes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // The table addresses are absolute: the allocation must start at kSmemBase.
  if (smem_addr(smem) != kSmemBase) {
    if (threadIdx.x == 0) atomicOr(&g_cc_error, 1u);
    return;
  }
  float* xs = reinterpret_cast<float*>(smem);
  float* part = reinterpret_cast<float*>(smem + S::kPartOff);
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = S::kXBytes / 4;
                    const int part_floats = (int)(seedlm_dynamic_smem_bytes() - S::kPartOff) / 4;)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lane8 = (uint32_t)(lane & 15) << 3;

  rep::fill_rep_tables<C, 0>(smem, threadIdx.x, blockDim.x);
  // Records and X may be the previous kernel's output: read them only now.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int g0 = (int)((int64_t)blockIdx.x * g.groups / gridDim.x);
  const int g1 = (int)((int64_t)(blockIdx.x + 1) * g.groups / gridDim.x);
  CcRecs<kRows> buf[kAhead + 1];
  for (int p0 = g0; p0 < g1; p0 += g.pass_groups) {
    const int p1 = min(p0 + g.pass_groups, g1);
    const int pass_rows = (p1 - p0) * kRows;
    // Warp w's sum for row t and X row m at part[(w * MB + m) * pass_rows + t].
    for (int i = threadIdx.x; i < pass_rows * MB * kWarps; i += blockDim.x)
      if (SEEDLM_IN_BOUNDS(g_check_flag, i, part_floats)) part[i] = 0.f;
    for (int sg = 0; sg < g.n_segs; ++sg) {
      const int s0 = sg * g.seg_spans;
      const int sl = min(g.seg_spans, g.n_spans - s0);
      const int items = (p1 - p0) * sl;
      const int i0 = (int)((int64_t)warp * items / kWarps);
      const int i1 = (int)((int64_t)(warp + 1) * items / kWarps);
      // Item cursor (grp, span) and load cursor (lgrp, lspan), kAhead items
      // ahead; the first records are in flight while X is staged.
      int grp = p0 + (i0 < i1 ? i0 / sl : 0), span = i0 < i1 ? i0 % sl : 0;
      int lgrp = grp, lspan = span;
#pragma unroll
      for (int k = 0; k < kAhead; ++k) {
        if (i0 + k < i1) load_recs<C, kRows>(buf[k], rec, eplane, g, lgrp, (s0 + lspan) * kSpan + lane);
        if (++lspan == sl) { lspan = 0; ++lgrp; }
      }
      if (g.n_segs > 1 || p0 == g0) stage_x<C, MB>(xs, X, is_bf16, g, s0, sl, vec);
      __syncthreads();  // X, tables and zeroed partials ready
      if (i0 < i1) {
        float2 acc[kRows][MB];
#pragma unroll
        for (int j = 0; j < kRows; ++j)
#pragma unroll
          for (int m = 0; m < MB; ++m) acc[j][m] = make_float2(0.f, 0.f);
        // kAhead + 1 record buffers, indexed by constants (the loop is
        // unrolled by kAhead + 1), so they stay in registers.
        for (int c2 = i0; c2 < i1; c2 += kAhead + 1) {
#pragma unroll
          for (int k = 0; k <= kAhead; ++k) {
            const int ci = c2 + k;
            if (ci < i1) {
              if (ci + kAhead < i1) {
                load_recs<C, kRows>(buf[(k + kAhead) % (kAhead + 1)], rec, eplane, g, lgrp,
                                    (s0 + lspan) * kSpan + lane);
                if (++lspan == sl) { lspan = 0; ++lgrp; }
              }
              const int ul = span * kSpan + lane;  // the lane's unit within the segment
              float2 xe[kE];
#pragma unroll
              for (int q = 0; q < kE / 2; ++q) {
                const int si = slot_index<C, MB>(ul, 2 * q);
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (SEEDLM_IN_BOUNDS(g_check_flag, si + 3, xs_floats)) v = *reinterpret_cast<const float4*>(xs + si);
                xe[2 * q] = make_float2(v.x, v.y);
                xe[2 * q + 1] = make_float2(v.z, v.w);
              }
              rebuild_and_dot<C, MB, kRows>(buf[k], xe, (s0 + span) * kSpan + lane, lane8, acc);
              const bool end_group = ++span == sl;
              if (end_group || ci + 1 == i1) {
                // The warp leaves the group: its sums into its own slots.
#pragma unroll
                for (int j = 0; j < kRows; ++j) {
#pragma unroll
                  for (int m = 0; m < MB; ++m) {
                    float s = acc[j][m].x + acc[j][m].y;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                    const int pi = (warp * MB + m) * pass_rows + (grp - p0) * kRows + j;
                    if (lane == 0 && SEEDLM_IN_BOUNDS(g_check_flag, pi, part_floats)) part[pi] += s;
                    acc[j][m] = make_float2(0.f, 0.f);
                  }
                }
              }
              if (end_group) { span = 0; ++grp; }
            }
          }
        }
      }
      __syncthreads();  // partials complete; X may be restaged
    }
    for (int i = threadIdx.x; i < pass_rows * MB; i += blockDim.x) {
      const int m = i / pass_rows, t = i - m * pass_rows;
      const int r = p0 * kRows + t;
      if (r < g.rows && m < g.M) {
        float sum = 0.f;
        for (int w = 0; w < kWarps; ++w) {
          const int pi = (w * MB + m) * pass_rows + t;
          if (SEEDLM_IN_BOUNDS(g_check_flag, pi, part_floats)) sum += part[pi];
        }
        if (SEEDLM_IN_BOUNDS(g_check_flag, (size_t)m * g.rows + r, (size_t)g.M * g.rows))
          Y[(size_t)m * g.rows + r] = sum;
      }
    }
    __syncthreads();  // partials read before the next pass clears them
  }
}

template <int C, int MB>
CcGeom make_geom(const seedlm_format& f, int M, int grid, const DeviceInfo& dev) {
  using S = CcSmem<C, MB>;
  CcGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.M = M;
  g.groups = (f.rows + S::kRows - 1) / S::kRows;
  g.n_spans = (f.nb + kSpan - 1) / kSpan;
  if (g.n_spans < 1) g.n_spans = 1;
  g.n_segs = (g.n_spans + S::kMaxSegSpans - 1) / S::kMaxSegSpans;
  g.seg_spans = (g.n_spans + g.n_segs - 1) / g.n_segs;
  const int64_t room = (int64_t)dev.max_smem_optin - S::kPartOff;
  const int max_cta_groups = (g.groups + grid - 1) / grid;
  int64_t pg = room > 0 ? room / S::kPartBytesPerGroup : 0;
  if (pg > max_cta_groups) pg = max_cta_groups;
  g.pass_groups = (int)pg;
  return g;
}

template <int C, int MB>
int launch_cc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
              const uint16_t* X, int is_bf16, int M, float* Y, cudaStream_t stream,
              const DeviceInfo& dev) {
  using S = CcSmem<C, MB>;
  const int groups = (f.rows + S::kRows - 1) / S::kRows;
  const int grid = groups < dev.num_sms ? groups : dev.num_sms;
  const CcGeom g = make_geom<C, MB>(f, M, grid, dev);
  if (g.pass_groups < 1) return SEEDLM_EUNSUPPORTED;
  const void* kern = (const void*)gemm_cc_kernel<C, MB>;
  int rc = allow_max_smem(kern, dev);
  if (rc) return rc;
  // 8-byte X loads: X 8-byte aligned and every row's start a multiple of 4 columns.
  const int vec = (reinterpret_cast<uintptr_t>(X) % 8 == 0) && (f.cols % 4 == 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = (size_t)S::kPartOff + (size_t)g.pass_groups * S::kPartBytesPerGroup;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {(void*)&rec, (void*)&eplane, (void*)&X, (void*)&is_bf16, (void*)&vec,
                  (void*)&Y, (void*)&g};
  cudaError_t err = cudaLaunchKernelExC(&cfg, kern, args);
  if (err != cudaSuccess) return record_cuda_error(err);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace

bool gemm_cc_applies(const seedlm_format& f, int M) {
  return M >= 2 && M <= kGemmCcMaxRows && f.rows > 0 && f.cols > 0 && f.C == 12;
}

int launch_gemm_cc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                   const uint16_t* X, int is_bf16, int M, float* Y, cudaStream_t stream,
                   const DeviceInfo& dev) {
  if (!gemm_cc_applies(f, M)) return SEEDLM_EUNSUPPORTED;
  return M <= 2 ? launch_cc<12, 2>(f, rec, eplane, X, is_bf16, M, Y, stream, dev)
                : launch_cc<12, 4>(f, rec, eplane, X, is_bf16, M, Y, stream, dev);
}

int read_and_clear_cc_error(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, g_cc_error, sizeof(v));
  if (err != cudaSuccess) return record_cuda_error(err);
  if (v) {
    err = cudaMemcpyToSymbol(g_cc_error, &zero, sizeof(zero));
    if (err != cudaSuccess) return record_cuda_error(err);
  }
  *out = v;
  return SEEDLM_OK;
}

}  // namespace seedlm
