// gemv.cu -- y = W x with W rebuilt block by block on the fly (batch 1).
//
// SeedLM inference (paperhub.cn review thread, authors' reply on how inference
// uses Eq (1)): the seed and coefficients of each block are read from memory,
// the block is rebuilt and consumed at once; W never exists in full precision.
//
// Work decomposition (one CTA of 16 warps per SM, persistent):
//   * x is converted to fp32 once per CTA into shared memory, zero-padded, in
//     a swizzled "record pair" layout: for records 2rp and 2rp+1 of a row the
//     x values of column c of both blocks sit side by side, so one packed
//     fp32x2 FMA consumes weight c of both blocks.  The XOR swizzle makes the
//     lanes of a quarter-warp hit distinct banks.
//   * A task is 4 rows x 32 record pairs (one pair per lane): the lane loads
//     the two records of each row (8 bytes, coalesced across the warp), keeps
//     the pair's x values in registers for all 4 rows, and accumulates four
//     fp32x2 row sums.
//   * A tile is G groups of 4 rows; its G * n_spans tasks are split evenly
//     over the 16 warps (G is chosen so the count divides by 16 when the
//     matrix is large enough).  Warp partial sums meet in shared memory and
//     are added in warp order, so every call gives the same bits.
//   * The next task's records are loaded before the current task is rebuilt.
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerTask = 4;
constexpr int kMaxGroups = 16;

struct GemvGeom {
  int rows, nb, rec_pitch, e_pitch, cols;
  int nbp;      // record pairs per row that hold data: ceil(nb / 2)
  int n_spans;  // ceil(nbp / 32)
  int groups;   // G: groups of 4 rows per tile
  int tiles;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Shared-memory map: [tables][partials kMaxGroups*4*kWarps floats][x slots].
template <int C>
struct Smem {
  static constexpr int kTableBytes = (C == 8) ? 2 * 256 * 4 : 2 * 256 * 8;
  static constexpr int kPartBytes = kMaxGroups * kRowsPerTask * kWarps * 4;
  static constexpr int kSlotFloats = (C == 8) ? 16 : 32;  // per record pair
  static constexpr int kHead = kTableBytes + kPartBytes;
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
  // Tables.
  if constexpr (C == 8) {
    uint32_t* t = reinterpret_cast<uint32_t*>(smem);
    for (int i = threadIdx.x; i < 512; i += kThreads)
      t[i] = (uint32_t)(i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256]);
  } else {
    uint2* t = reinterpret_cast<uint2*>(smem);
    for (int i = threadIdx.x; i < 512; i += kThreads) {
      uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
      t[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
    }
  }
  // Partials.
  float* part = reinterpret_cast<float*>(smem + Smem<C>::kTableBytes);
  for (int i = threadIdx.x; i < kMaxGroups * kRowsPerTask * kWarps; i += kThreads) part[i] = 0.f;
  // x, zero-padded to n_spans * 32 record pairs.
  float* xs = reinterpret_cast<float*>(smem + Smem<C>::kHead);
  const int ncols_pad = g.n_spans * 32 * 2 * C;
  for (int j = threadIdx.x; j < ncols_pad; j += kThreads) {
    int rp = j / (2 * C);
    int w = j - rp * 2 * C;
    int h = w / C;
    int c = w - h * C;
    float v = j < g.cols ? act_to_float(x[j], is_bf16) : 0.f;
    xs[x_slot_index<C>(rp, c, h)] = v;
  }
}

// ---------------------------------------------------------------- C = 8

struct RecPairC8 {
  uint2 r[kRowsPerTask];
};

__device__ __forceinline__ void load_task_c8(RecPairC8& o, const uint32_t* __restrict__ rec,
                                             const GemvGeom& g, int row0, int rp) {
#pragma unroll
  for (int j = 0; j < kRowsPerTask; ++j) {
    int r = row0 + j;
    if (r < g.rows && 2 * rp < g.rec_pitch)
      o.r[j] = ld_stream_u2(rec + (size_t)r * g.rec_pitch + 2 * rp);
    else
      o.r[j] = make_uint2(0u, 0u);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
gemv_c8_kernel(const uint32_t* __restrict__ rec, const uint16_t* __restrict__ x, int is_bf16,
               float* __restrict__ y, GemvGeom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  stage_x_and_tables<8>(smem, x, is_bf16, g);
  __syncthreads();
  const uint32_t* t_lo = reinterpret_cast<const uint32_t*>(smem);
  const uint32_t* t_hi = t_lo + 256;
  float* part = reinterpret_cast<float*>(smem + Smem<8>::kTableBytes);
  const float* xs = reinterpret_cast<const float*>(smem + Smem<8>::kHead);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int swz = (lane >> 1) & 3;
  const int tasks = g.groups * g.n_spans;
  const int t_begin = warp * tasks / kWarps, t_end = (warp + 1) * tasks / kWarps;

  for (int tile = blockIdx.x; tile < g.tiles; tile += gridDim.x) {
    const int tile_row0 = tile * g.groups * kRowsPerTask;
    RecPairC8 cur, nxt;
    if (t_begin < t_end) {
      int grp = t_begin / g.n_spans, span = t_begin - grp * g.n_spans;
      load_task_c8(cur, rec, g, tile_row0 + grp * kRowsPerTask, span * 32 + lane);
    }
    float2 acc[kRowsPerTask];
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j) acc[j] = make_float2(0.f, 0.f);
    for (int t = t_begin; t < t_end; ++t) {
      const int grp = t / g.n_spans, span = t - grp * g.n_spans;
      const int rp = span * 32 + lane;
      if (t + 1 < t_end) {
        int g2 = (t + 1) / g.n_spans, s2 = (t + 1) - g2 * g.n_spans;
        load_task_c8(nxt, rec, g, tile_row0 + g2 * kRowsPerTask, s2 * 32 + lane);
      }
      // x pairs of this record pair: xp[c] = (x[16 rp + c], x[16 rp + 8 + c]).
      float2 xp[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float4 v = *reinterpret_cast<const float4*>(xs + rp * 16 + ((i ^ swz) << 2));
        xp[2 * i] = make_float2(v.x, v.y);
        xp[2 * i + 1] = make_float2(v.z, v.w);
      }
#pragma unroll
      for (int j = 0; j < kRowsPerTask; ++j) {
        const BlockC8 A = decode_c8(cur.r[j].x, t_lo, t_hi);
        const BlockC8 B = decode_c8(cur.r[j].y, t_lo, t_hi);
        const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
        float2 a = acc[j];
#define SEEDLM_C8_STEP(c)                                                               \
  {                                                                                     \
    float2 w = make_float2(__int_as_float(weight_bits_c8<c>(A)),                        \
                           __int_as_float(weight_bits_c8<c>(B)));                       \
    a = __ffma2_rn(__fadd2_rn(w, negm), xp[c], a);                                      \
  }
        SEEDLM_C8_STEP(0) SEEDLM_C8_STEP(1) SEEDLM_C8_STEP(2) SEEDLM_C8_STEP(3)
        SEEDLM_C8_STEP(4) SEEDLM_C8_STEP(5) SEEDLM_C8_STEP(6) SEEDLM_C8_STEP(7)
#undef SEEDLM_C8_STEP
        acc[j] = a;
      }
      // Flush when the group changes or the warp's range ends.
      const bool last = (t + 1 == t_end) || ((t + 1) / g.n_spans != grp);
      if (last) {
#pragma unroll
        for (int j = 0; j < kRowsPerTask; ++j) {
          float s = warp_sum(acc[j].x + acc[j].y);
          if (lane == 0) part[(grp * kRowsPerTask + j) * kWarps + warp] = s;
          acc[j] = make_float2(0.f, 0.f);
        }
      }
      cur = nxt;
    }
    __syncthreads();
    const int trows = g.groups * kRowsPerTask;
    if (threadIdx.x < trows) {
      float s = 0.f;
      float* p = part + threadIdx.x * kWarps;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        s += p[w];
        p[w] = 0.f;
      }
      const int r = tile_row0 + threadIdx.x;
      if (r < g.rows) y[r] = s;
    }
    __syncthreads();
  }
}

// --------------------------------------------------------------- C = 12

struct RecPairC12 {
  uint2 r[kRowsPerTask];
  uint32_t e[kRowsPerTask];  // exponent byte of the pair (both nibbles)
};

__device__ __forceinline__ void load_task_c12(RecPairC12& o, const uint32_t* __restrict__ rec,
                                              const uint8_t* __restrict__ eplane,
                                              const GemvGeom& g, int row0, int rp) {
#pragma unroll
  for (int j = 0; j < kRowsPerTask; ++j) {
    int r = row0 + j;
    if (r < g.rows && 2 * rp < g.rec_pitch) {
      o.r[j] = ld_stream_u2(rec + (size_t)r * g.rec_pitch + 2 * rp);
      o.e[j] = rp < g.e_pitch ? ld_stream_u8(eplane + (size_t)r * g.e_pitch + rp) : 0u;
    } else {
      o.r[j] = make_uint2(0u, 0u);
      o.e[j] = 0u;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
gemv_c12_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
                const uint16_t* __restrict__ x, int is_bf16, float* __restrict__ y, GemvGeom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  stage_x_and_tables<12>(smem, x, is_bf16, g);
  __syncthreads();
  const uint2* t_lo = reinterpret_cast<const uint2*>(smem);
  const uint2* t_hi = t_lo + 256;
  float* part = reinterpret_cast<float*>(smem + Smem<12>::kTableBytes);
  const float* xs = reinterpret_cast<const float*>(smem + Smem<12>::kHead);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int swz = lane & 7;
  const int tasks = g.groups * g.n_spans;
  const int t_begin = warp * tasks / kWarps, t_end = (warp + 1) * tasks / kWarps;

  for (int tile = blockIdx.x; tile < g.tiles; tile += gridDim.x) {
    const int tile_row0 = tile * g.groups * kRowsPerTask;
    RecPairC12 cur, nxt;
    if (t_begin < t_end) {
      int grp = t_begin / g.n_spans, span = t_begin - grp * g.n_spans;
      load_task_c12(cur, rec, eplane, g, tile_row0 + grp * kRowsPerTask, span * 32 + lane);
    }
    float2 acc[kRowsPerTask];
#pragma unroll
    for (int j = 0; j < kRowsPerTask; ++j) acc[j] = make_float2(0.f, 0.f);
    for (int t = t_begin; t < t_end; ++t) {
      const int grp = t / g.n_spans, span = t - grp * g.n_spans;
      const int rp = span * 32 + lane;
      if (t + 1 < t_end) {
        int g2 = (t + 1) / g.n_spans, s2 = (t + 1) - g2 * g.n_spans;
        load_task_c12(nxt, rec, eplane, g, tile_row0 + g2 * kRowsPerTask, s2 * 32 + lane);
      }
      float2 xp[12];
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        float4 v = *reinterpret_cast<const float4*>(xs + rp * 32 + ((i ^ swz) << 2));
        xp[2 * i] = make_float2(v.x, v.y);
        xp[2 * i + 1] = make_float2(v.z, v.w);
      }
#pragma unroll
      for (int j = 0; j < kRowsPerTask; ++j) {
        const BlockC12 A = decode_c12(cur.r[j].x, cur.e[j], t_lo, t_hi);
        const BlockC12 B = decode_c12(cur.r[j].y, cur.e[j] >> 4, t_lo, t_hi);
        const float2 negm = make_float2(__uint_as_float(A.negm), __uint_as_float(B.negm));
        float2 a = acc[j];
#define SEEDLM_C12_STEP(c)                                                              \
  {                                                                                     \
    float2 w = make_float2(__int_as_float(weight_bits_c12<c>(A)),                       \
                           __int_as_float(weight_bits_c12<c>(B)));                      \
    a = __ffma2_rn(__fadd2_rn(w, negm), xp[c], a);                                      \
  }
        SEEDLM_C12_STEP(0) SEEDLM_C12_STEP(1) SEEDLM_C12_STEP(2) SEEDLM_C12_STEP(3)
        SEEDLM_C12_STEP(4) SEEDLM_C12_STEP(5) SEEDLM_C12_STEP(6) SEEDLM_C12_STEP(7)
        SEEDLM_C12_STEP(8) SEEDLM_C12_STEP(9) SEEDLM_C12_STEP(10) SEEDLM_C12_STEP(11)
#undef SEEDLM_C12_STEP
        acc[j] = a;
      }
      const bool last = (t + 1 == t_end) || ((t + 1) / g.n_spans != grp);
      if (last) {
#pragma unroll
        for (int j = 0; j < kRowsPerTask; ++j) {
          float s = warp_sum(acc[j].x + acc[j].y);
          if (lane == 0) part[(grp * kRowsPerTask + j) * kWarps + warp] = s;
          acc[j] = make_float2(0.f, 0.f);
        }
      }
      cur = nxt;
    }
    __syncthreads();
    const int trows = g.groups * kRowsPerTask;
    if (threadIdx.x < trows) {
      float s = 0.f;
      float* p = part + threadIdx.x * kWarps;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        s += p[w];
        p[w] = 0.f;
      }
      const int r = tile_row0 + threadIdx.x;
      if (r < g.rows) y[r] = s;
    }
    __syncthreads();
  }
}

int gcd_int(int a, int b) {
  while (b) {
    int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

GemvGeom make_geom(const seedlm_format& f, int num_sms) {
  GemvGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.nbp = (f.nb + 1) / 2;
  g.n_spans = (g.nbp + 31) / 32;
  if (g.n_spans < 1) g.n_spans = 1;
  // Enough groups per tile that the tile's tasks divide over the 16 warps,
  // but not so many that there are fewer tiles than SMs.
  int want = kWarps / gcd_int(kWarps, g.n_spans);
  int groups_total = (f.rows + kRowsPerTask - 1) / kRowsPerTask;
  int cap = groups_total / (num_sms > 0 ? num_sms : 1);
  if (cap < 1) cap = 1;
  g.groups = want < cap ? want : cap;
  if (g.groups > kMaxGroups) g.groups = kMaxGroups;
  g.tiles = (groups_total + g.groups - 1) / g.groups;
  return g;
}

}  // namespace

size_t gemv_smem_bytes(const seedlm_format& f) {
  int nbp = (f.nb + 1) / 2;
  int n_spans = (nbp + 31) / 32;
  if (n_spans < 1) n_spans = 1;
  if (f.C == 8) return (size_t)Smem<8>::kHead + (size_t)n_spans * 32 * Smem<8>::kSlotFloats * 4;
  return (size_t)Smem<12>::kHead + (size_t)n_spans * 32 * Smem<12>::kSlotFloats * 4;
}

int launch_gemv(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                const DeviceInfo& dev) {
  GemvGeom g = make_geom(f, dev.num_sms);
  size_t smem = gemv_smem_bytes(f);
  if (smem > (size_t)dev.max_smem_optin) return SEEDLM_EUNSUPPORTED;
  int grid = g.tiles < dev.num_sms ? g.tiles : dev.num_sms;
  if (grid < 1) return SEEDLM_OK;
  if (f.C == 8) {
    int rc_attr = allow_max_smem((const void*)gemv_c8_kernel, dev);
    if (rc_attr) return rc_attr;
    gemv_c8_kernel<<<grid, kThreads, smem, stream>>>(rec, x, is_bf16, y, g);
  } else {
    int rc_attr = allow_max_smem((const void*)gemv_c12_kernel, dev);
    if (rc_attr) return rc_attr;
    gemv_c12_kernel<<<grid, kThreads, smem, stream>>>(rec, eplane, x, is_bf16, y, g);
  }
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace seedlm
