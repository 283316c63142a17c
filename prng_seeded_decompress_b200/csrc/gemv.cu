// gemv.cu -- y = W x with W rebuilt block by block on the fly (batch 1).
//
// SeedLM inference (paperhub.cn review thread, authors' reply on how inference
// uses Eq (1)): the seed and coefficients of each block are read from memory,
// the block is rebuilt and consumed at once; W never exists in full precision.
//
// Work decomposition (one CTA per SM, up to 16 warps, persistent):
//   * x is converted to fp32 once per CTA into shared memory, zero-padded, in
//     a swizzled "record pair" layout: for records 2rp and 2rp+1 of a row the
//     x values of column c of both blocks sit side by side, so one packed
//     fp32x2 FMA consumes weight c of both blocks.  The XOR swizzle makes the
//     lanes of a quarter-warp hit distinct banks.
//   * An item is a group of 4 rows x one span of 32 record pairs (one pair
//     per lane): the lane loads the two records of each row (8 bytes,
//     coalesced across the warp), keeps the pair's x values in registers for
//     all 4 rows, and accumulates one fp32x2 sum per row.  Record sets are
//     loaded two items ahead of the one being rebuilt.
//   * Each CTA owns a contiguous range of row groups and splits its items
//     evenly over its warps, so every SM and every warp gets the same work
//     to within one item.  Row sums are reduced with warp shuffles and then
//     across warps in shared memory, in a fixed order, so every call gives
//     the same bits.
//   * Launched with programmatic stream serialization: the first record
//     loads are issued before griddepcontrol.wait, so back-to-back GEMVs
//     overlap one kernel's tail with the next one's prologue; x is read only
//     after the wait.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

// 1: take the C = 8 coefficient decode from two 256-entry shared tables;
// 0: compute it with byte arithmetic and dp2a.
#ifndef SEEDLM_GEMV_COEF_TABLES
#define SEEDLM_GEMV_COEF_TABLES 1
#endif

namespace seedlm {

SEEDLM_CHECK_FLAG(gemv)

namespace {

// Warps per CTA (one CTA per SM) and record sets in flight ahead of the one
// being rebuilt.  C = 8 runs 24 warps with one set ahead; C = 12 needs more
// registers per lane (four dp2a windows per weight) and spills at 24 warps, so
// it keeps 16 warps with two sets ahead.
template <int C>
struct Tune {
  static constexpr int kWarps = (C == 8) ? 24 : 16;
  static constexpr int kPrefetch = (C == 8) ? 1 : 2;
};
constexpr int kRowsPerTask = 4;
constexpr int kMinWarps = 8;      // warps per CTA however few items it has
constexpr int kMaxGroups = 128;  // row groups per partial-sum pass (fewer if x needs the room)

struct GemvGeom {
  int rows, cols, nb, rec_pitch, e_pitch;
  int n_spans;      // ceil(ceil(nb / 2) / 32): 32 record pairs (one per lane) per span
  int groups;       // ceil(rows / 4)
  int pass_groups;  // row groups per partial-sum pass (<= kMaxGroups)
  int x_off;        // byte offset of the x slots in shared memory
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Shared-memory map: [jump tables][partial sums][x slots].  The partial-sum
// buffer holds pass_groups row groups; x starts at x_off (both chosen by the
// launcher so that x fits).
template <int C>
struct Smem {
  // C = 8: jump tables (2 KB) + coefficient tables (4 KB); C = 12: jump tables.
  static constexpr int kJumpBytes = (C == 8) ? 2 * 256 * 4 : 2 * 256 * 8;
  static constexpr int kTableBytes = (C == 8) ? kJumpBytes + 2 * 256 * 8 : kJumpBytes;
  static constexpr int kPartBytesPerGroup = kRowsPerTask * Tune<C>::kWarps * 4;
  static constexpr int kSlotFloats = (C == 8) ? 16 : 32;  // per record pair
};

template <int C>
__device__ __forceinline__ int x_slot_index(int rp, int c, int h) {
  // Float index of column (record 2rp+h, weight c) in the swizzled layout.
  if constexpr (C == 8) {
    return rp * 16 + (((c >> 1) ^ ((rp >> 1) & 3)) << 2) + ((c & 1) << 1) + h;
  } else {
    return rp * 32 + (((c >> 1) ^ (rp & 7)) << 2) + ((c & 1) << 1) + h;
  }
}

template <int C>
__device__ void stage_x_and_tables(unsigned char* smem, const uint16_t* __restrict__ x, int is_bf16,
                                   const GemvGeom& g) {
  if constexpr (C == 8) {
    uint32_t* t = reinterpret_cast<uint32_t*>(smem);
    for (int i = threadIdx.x; i < 512; i += blockDim.x)
      t[i] = (uint32_t)(i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256]);
    uint2* tq = reinterpret_cast<uint2*>(smem + Smem<8>::kJumpBytes);
    fill_coef_tables_c8(tq, tq + 256, threadIdx.x, blockDim.x);
  } else {
    uint2* t = reinterpret_cast<uint2*>(smem);
    for (int i = threadIdx.x; i < 512; i += blockDim.x) {
      uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
      t[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
    }
  }
  // x, zero-padded to n_spans * 32 record pairs.
  float* xs = reinterpret_cast<float*>(smem + g.x_off);
  const int ncols_pad = g.n_spans * 32 * 2 * C;
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = (seedlm_dynamic_smem_bytes() - g.x_off) / 4;)
  for (int j = threadIdx.x; j < ncols_pad; j += blockDim.x) {
    int rp = j / (2 * C);
    int w = j - rp * 2 * C;
    int h = w / C;
    int c = w - h * C;
    float v = j < g.cols ? act_to_float(x[j], is_bf16) : 0.f;
    const int si = x_slot_index<C>(rp, c, h);
    if (SEEDLM_IN_BOUNDS(g_check_flag, si, xs_floats)) xs[si] = v;
  }
}

// The records one lane needs for one (row group, span) item: the pair of
// blocks (2rp, 2rp+1) in each of the group's 4 rows, plus for C = 12 the
// exponent byte of the pair.  Rows past `rows` and pairs past the row pitch
// read as zero records (their x is zero, so they add nothing).
template <int C>
struct RecSet {
  uint2 r[kRowsPerTask];
  uint32_t e[C == 12 ? kRowsPerTask : 1];
};

template <int C>
__device__ __forceinline__ void load_set(RecSet<C>& o, const uint32_t* __restrict__ rec,
                                         const uint8_t* __restrict__ eplane, const GemvGeom& g,
                                         int grp, int span, int lane) {
  const int row0 = grp * kRowsPerTask;
  const int rp = span * 32 + lane;
  const bool pair_ok = 2 * rp < g.rec_pitch;
  const uint32_t* p = rec + (size_t)row0 * g.rec_pitch + 2 * rp;
#pragma unroll
  for (int j = 0; j < kRowsPerTask; ++j) {
    // The pair's second record is the last word read.
    const bool ok = pair_ok && row0 + j < g.rows &&
                    SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(row0 + j) * g.rec_pitch + 2 * rp + 1,
                                     (size_t)g.rows * g.rec_pitch);
    o.r[j] = ok ? ld_stream_u2(p + (size_t)j * g.rec_pitch) : make_uint2(0u, 0u);
    if constexpr (C == 12)
      o.e[j] = (ok && rp < g.e_pitch &&
                SEEDLM_IN_BOUNDS(g_check_flag, (size_t)(row0 + j) * g.e_pitch + rp,
                                 (size_t)g.rows * g.e_pitch))
                   ? ld_stream_u8(eplane + (size_t)(row0 + j) * g.e_pitch + rp)
                   : 0u;
  }
}

// Rebuild the lane's 2 x C weights of each of the 4 rows and accumulate
// w * x into one fp32x2 sum per row.
template <int C>
__device__ __forceinline__ void rebuild_and_dot(const RecSet<C>& cur, const float* __restrict__ xs,
                                                int rp, int swz, const void* t_lo, const void* t_hi,
                                                float2 (&acc)[kRowsPerTask]) {
  float2 xp[C];
#pragma unroll
  for (int i = 0; i < C / 2; ++i) {
    float4 v = *reinterpret_cast<const float4*>(xs + rp * Smem<C>::kSlotFloats + ((i ^ swz) << 2));
    xp[2 * i] = make_float2(v.x, v.y);
    xp[2 * i + 1] = make_float2(v.z, v.w);
  }
#pragma unroll
  for (int j = 0; j < kRowsPerTask; ++j) {
    float2 a = acc[j];
    if constexpr (C == 8) {
      const uint32_t* tl = static_cast<const uint32_t*>(t_lo);
      const uint32_t* th = static_cast<const uint32_t*>(t_hi);
#if SEEDLM_GEMV_COEF_TABLES
      const uint2* tq1 = reinterpret_cast<const uint2*>(th + 256);
      const BlockC8 A = decode_c8_tab(cur.r[j].x, tl, th, tq1, tq1 + 256);
      const BlockC8 B = decode_c8_tab(cur.r[j].y, tl, th, tq1, tq1 + 256);
#else
      const BlockC8 A = decode_c8(cur.r[j].x, tl, th);
      const BlockC8 B = decode_c8(cur.r[j].y, tl, th);
#endif
      const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
#define SEEDLM_C8_STEP(c)                                                        \
  {                                                                              \
    float2 w = make_float2(__int_as_float(weight_bits_c8<c>(A)),                 \
                           __int_as_float(weight_bits_c8<c>(B)));                \
    a = __ffma2_rn(__fadd2_rn(w, negm), xp[c], a);                               \
  }
      SEEDLM_C8_STEP(0) SEEDLM_C8_STEP(1) SEEDLM_C8_STEP(2) SEEDLM_C8_STEP(3)
      SEEDLM_C8_STEP(4) SEEDLM_C8_STEP(5) SEEDLM_C8_STEP(6) SEEDLM_C8_STEP(7)
#undef SEEDLM_C8_STEP
    } else {
      const uint2* tl = static_cast<const uint2*>(t_lo);
      const uint2* th = static_cast<const uint2*>(t_hi);
      const BlockC12 A = decode_c12(cur.r[j].x, cur.e[j], tl, th);
      const BlockC12 B = decode_c12(cur.r[j].y, cur.e[j] >> 4, tl, th);
      const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
#define SEEDLM_C12_STEP(c)                                                       \
  {                                                                              \
    float2 w = make_float2(__int_as_float(weight_bits_c12<c>(A)),                \
                           __int_as_float(weight_bits_c12<c>(B)));               \
    a = __ffma2_rn(__fadd2_rn(w, negm), xp[c], a);                               \
  }
      SEEDLM_C12_STEP(0) SEEDLM_C12_STEP(1) SEEDLM_C12_STEP(2) SEEDLM_C12_STEP(3)
      SEEDLM_C12_STEP(4) SEEDLM_C12_STEP(5) SEEDLM_C12_STEP(6) SEEDLM_C12_STEP(7)
      SEEDLM_C12_STEP(8) SEEDLM_C12_STEP(9) SEEDLM_C12_STEP(10) SEEDLM_C12_STEP(11)
#undef SEEDLM_C12_STEP
    }
    acc[j] = a;
  }
}

// CTA b owns the contiguous row groups [g0, g1) (sizes differ by at most
// one group); its (group, span) items are split into equal contiguous ranges,
// one per warp.  A warp walks its range with record sets loaded Tune<C>::kPrefetch
// items ahead (across group boundaries), and whenever it leaves a group it
// reduces its 4 row sums with shuffles into shared memory.  After a barrier
// the partial sums of each row are added in warp order -- the same order on
// every call -- and written.  Groups are processed in passes of at most
// pass_groups so the partial-sum buffer stays small.
template <int C>
__global__ void __launch_bounds__(Tune<C>::kWarps * 32, 1)
gemv_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
            const uint16_t* __restrict__ x, int is_bf16, float* __restrict__ y, GemvGeom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  const void* t_lo = smem;
  const void* t_hi = smem + Smem<C>::kJumpBytes / 2;
  float* part = reinterpret_cast<float*>(smem + Smem<C>::kTableBytes);
  const float* xs = reinterpret_cast<const float*>(smem + g.x_off);
  SEEDLM_CHECK_ONLY(const unsigned int xs_floats = (seedlm_dynamic_smem_bytes() - g.x_off) / 4;
                    const int part_floats = (g.x_off - Smem<C>::kTableBytes) / 4;)

  const int nw = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int swz = (C == 8) ? ((lane >> 1) & 3) : (lane & 7);
  const int g0 = (int)((int64_t)blockIdx.x * g.groups / gridDim.x);
  const int g1 = (int)((int64_t)(blockIdx.x + 1) * g.groups / gridDim.x);

  bool first_pass = true;
  for (int p0 = g0; p0 < g1; p0 += g.pass_groups) {
    const int p1 = min(p0 + g.pass_groups, g1);
    const int items = (p1 - p0) * g.n_spans;
    const int i0 = (int)((int64_t)warp * items / nw), i1 = (int)((int64_t)(warp + 1) * items / nw);
    // The first record sets are requested before anything else: they do not
    // depend on x, so their latency overlaps the staging of x (and, with
    // programmatic dependent launch, the tail of the previous kernel).
    int grp = p0 + (i0 < i1 ? i0 / g.n_spans : 0), span = i0 < i1 ? i0 % g.n_spans : 0;
    int lgrp = grp, lspan = span, li = i0;
    RecSet<C> buf[Tune<C>::kPrefetch + 1];
#pragma unroll
    for (int k = 0; k <= Tune<C>::kPrefetch; ++k) {
      if (li < i1) load_set<C>(buf[k], rec, eplane, g, lgrp, lspan, lane);
      ++li;
      if (++lspan == g.n_spans) { lspan = 0; ++lgrp; }
    }
    if (first_pass) {
      // x may be the previous kernel's output: wait for it only now.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      stage_x_and_tables<C>(smem, x, is_bf16, g);
      first_pass = false;
    }
    for (int i = threadIdx.x; i < (p1 - p0) * kRowsPerTask * nw; i += blockDim.x)
      if (SEEDLM_IN_BOUNDS(g_check_flag, i, part_floats)) part[i] = 0.f;
    __syncthreads();  // x, tables and zeroed partials ready
    if (i0 < i1) {
      float2 acc[kRowsPerTask];
#pragma unroll
      for (int j = 0; j < kRowsPerTask; ++j) acc[j] = make_float2(0.f, 0.f);
      int ci = i0;
      bool done = false;
      while (!done) {
#pragma unroll
        for (int k = 0; k <= Tune<C>::kPrefetch; ++k) {
          if (!done) {
            // Every x slot of the lane's record pair lies in its kSlotFloats row.
            if (SEEDLM_IN_BOUNDS(g_check_flag,
                                 (span * 32 + lane + 1) * Smem<C>::kSlotFloats - 1, xs_floats))
              rebuild_and_dot<C>(buf[k], xs, span * 32 + lane, swz, t_lo, t_hi, acc);
            if (li < i1) load_set<C>(buf[k], rec, eplane, g, lgrp, lspan, lane);
            ++li;
            if (++lspan == g.n_spans) { lspan = 0; ++lgrp; }
            ++ci;
            const bool end_group = (++span == g.n_spans);
            if (end_group || ci == i1) {
#pragma unroll
              for (int j = 0; j < kRowsPerTask; ++j) {
                const float s = warp_sum(acc[j].x + acc[j].y);
                const int pi = ((grp - p0) * kRowsPerTask + j) * nw + warp;
                if (lane == 0 && SEEDLM_IN_BOUNDS(g_check_flag, pi, part_floats)) part[pi] = s;
                acc[j] = make_float2(0.f, 0.f);
              }
              if (end_group) { span = 0; ++grp; }
              done = (ci == i1);
            }
          }
        }
      }
    }
    __syncthreads();
    if (p1 == g1) {
      // The next kernel in the stream may start its prologue now.
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    }
    for (int t = threadIdx.x; t < (p1 - p0) * kRowsPerTask; t += blockDim.x) {
      const int r = p0 * kRowsPerTask + t;
      if (r < g.rows) {
        float s = 0.f;
        for (int w = 0; w < nw; ++w) s += part[t * nw + w];
        if (SEEDLM_IN_BOUNDS(g_check_flag, r, g.rows)) y[r] = s;
      }
    }
    __syncthreads();  // partials read before the next pass clears them
  }
}

// Shared memory of one CTA for a given pass size.
template <int C>
size_t smem_for(int n_spans, int pass_groups) {
  return (size_t)Smem<C>::kTableBytes + (size_t)pass_groups * Smem<C>::kPartBytesPerGroup +
         (size_t)n_spans * 32 * Smem<C>::kSlotFloats * 4;
}

// The geometry, with the largest partial-sum pass (<= kMaxGroups, halving)
// that leaves room for x; pass_groups = 0 if x alone does not fit.
template <int C>
GemvGeom make_geom(const seedlm_format& f, int max_smem) {
  GemvGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.n_spans = ((f.nb + 1) / 2 + 31) / 32;
  if (g.n_spans < 1) g.n_spans = 1;
  g.groups = (f.rows + kRowsPerTask - 1) / kRowsPerTask;
  g.pass_groups = kMaxGroups;
  while (g.pass_groups > 0 && smem_for<C>(g.n_spans, g.pass_groups) > (size_t)max_smem)
    g.pass_groups >>= 1;
  g.x_off = Smem<C>::kTableBytes + g.pass_groups * Smem<C>::kPartBytesPerGroup;
  return g;
}

}  // namespace

size_t gemv_smem_bytes(const seedlm_format& f, int max_smem) {
  if (f.C == 8) {
    const GemvGeom g = make_geom<8>(f, max_smem);
    return g.pass_groups ? smem_for<8>(g.n_spans, g.pass_groups) : 0;
  }
  const GemvGeom g = make_geom<12>(f, max_smem);
  return g.pass_groups ? smem_for<12>(g.n_spans, g.pass_groups) : 0;
}

int launch_gemv(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                const DeviceInfo& dev) {
  const GemvGeom g = (f.C == 8) ? make_geom<8>(f, dev.max_smem_optin)
                                : make_geom<12>(f, dev.max_smem_optin);
  if (g.pass_groups == 0) return SEEDLM_EUNSUPPORTED;  // x does not fit in shared memory
  const size_t smem = gemv_smem_bytes(f, dev.max_smem_optin);
  if (g.groups < 1) return SEEDLM_OK;
  // One CTA per SM (at most one per row group); fewer warps per CTA when
  // each CTA has only a few (group, span) items, so small matrices still
  // spread over all SMs.
  int grid = g.groups < dev.num_sms ? g.groups : dev.num_sms;
  int items_per_cta = (g.groups + grid - 1) / grid * g.n_spans;
  const int max_warps = (f.C == 8) ? Tune<8>::kWarps : Tune<12>::kWarps;
  int wpc = items_per_cta < max_warps ? items_per_cta : max_warps;
  // At least 8 warps: on small matrices the CTA's setup (x and the tables
  // into shared memory) outweighs its one or two items, and warps without
  // items still share it.
  if (wpc < kMinWarps) wpc = kMinWarps;
  const void* kern = (f.C == 8) ? (const void*)gemv_kernel<8> : (const void*)gemv_kernel<12>;
  int rc = allow_max_smem(kern, dev);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(wpc * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = (f.C == 8)
                        ? cudaLaunchKernelEx(&cfg, gemv_kernel<8>, rec, eplane, x, is_bf16, y, g)
                        : cudaLaunchKernelEx(&cfg, gemv_kernel<12>, rec, eplane, x, is_bf16, y, g);
  if (err != cudaSuccess) return record_cuda_error(err);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace seedlm
