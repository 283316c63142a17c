// gemv_amort.cu -- y = W x for tall 3-bit matrices (C = 12, P = 4), with the
// x-dependent part of every block's dot product taken from per-column-block
// tables shared by all rows.
//
// SeedLM rebuilds each block as W_blk = U t from the seed's LFSR states and
// multiplies it with the activations (paperhub.cn review thread, Eq (1) and
// the authors' reply on how inference uses s and t).  The dot of block b
// with its 12 activations is linear in the block's stream bits:
//
//   sum_c x_c w_c = 2^-e (sum_p q_p S_p - (sum_p q_p) X),
//   S_p = 2^-15 sum_c x_c state_{12p+c} = sum_{m=0..26} bit_{12p+m} X~_m,
//   X~_m = sum_c x_c 2^(m-c-15) (0 <= m - c <= 15),  X = sum_c x_c,
//
// where state_j is stream bits [j, j+16) (the 2^-15 keeps X~ within the
// range of x: |X~_m| <= sum |x_c|).  Cutting the 27 bits behind each S_p into
// four bytes gives S_p = T0[B0] + T1[B1] + T2[B2] + T3[B3] with
// T_j[v] = sum_k bit_k(v) X~_{8j+k}: 16 table lookups per block instead of
// 48 dp2a.  The tables depend on x only, so a CTA builds them once per strip
// of 32 column blocks and every row it owns reuses them.
//
//   * Lane l of a warp takes column block 32s + l of strip s: the tables
//     are interleaved by lane (row v holds entry v of the 32 column blocks
//     side by side, 128 bytes per table, two tables per 256-byte row), so
//     lane l always reads its own bank, every lookup is one conflict-free
//     wavefront, and its address is one prmt of the stream byte next to the
//     lane's offset.
//     T0/T1 and T2/T3 take 64 KB each, the lane-replicated stream jump
//     tables 64 more.
//   * A CTA owns up to 256 consecutive rows; warp w takes rows w, w + 16, ...
//     and keeps one running sum per row in registers across all strips, so
//     each row is reduced across the warp once, at the end (in a fixed
//     order: the result does not depend on timing).  A strip's records of
//     the warp's rows are requested before its tables are built (a variant
//     that requested them one strip ahead measured slower: the registers
//     it takes cost more than the latency it hides).
//
// Arithmetic: fp32 throughout (the tables' sums, S_p, the coefficient
// products); it meets the library's 1e-5 * sum |w x| bound with room to
// spare.  Used where a CTA has at least 128 rows (below that the tables'
// build outweighs what they save; gemv.cu serves those shapes).
#include <cuda_runtime.h>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"

namespace seedlm {

SEEDLM_CHECK_FLAG(gemv_amort)

namespace {

__device__ unsigned int g_amort_error = 0;

constexpr int kWarps = 16;
constexpr int kMaxRowsPerWarp = 16;  // rows a warp keeps sums for
constexpr int kMinRowsPerCta = 128;
constexpr int kStrip = 32;           // column blocks per strip (one per lane)

// Absolute shared addresses (the dynamic allocation starts at kBase).  A
// lookup address is (byte << 8) | lane offset, in [0, 0x10000), plus the
// table base in the load's immediate.
constexpr uint32_t kBase = 1024;
constexpr uint32_t kT01 = kBase;             // T0 (bytes 0..127 of a row), T1 (128..255)
constexpr uint32_t kT23 = kBase + 0x10000;   // T2, T3
constexpr uint32_t kJump = kBase + 0x20000;  // stream jump tables, 8-byte entries
constexpr uint32_t kXsum = kBase + 0x30000;  // the strip's 32 column-block sums
constexpr int kSmemBytes = (int)(kXsum + 128 - kBase);

template <uint32_t OFF>
__device__ __forceinline__ float ldsf(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF));
  return v;
}

template <uint32_t OFF>
__device__ __forceinline__ uint2 ldsu2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
  return v;
}

__device__ __forceinline__ void stsf(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// (byte K of w) << 8 | lane4.
template <int K>
__device__ __forceinline__ uint32_t row_addr(uint32_t w, uint32_t lane4) {
  return prmt<(0x5504u | ((uint32_t)K << 4))>(w, lane4);
}

struct AmortGeom {
  int rows, cols, nb, rec_pitch, e_pitch;
  int rows_per_cta;
  int strips;
};

// What a thread needs of one strip: the records of its warp's rows at its
// lane's block, their exponent nibbles (eight per word), and, for the table
// build, the 12 activations of column block (thread % 32) as 16-bit pairs.
struct StripIn {
  uint32_t r[kMaxRowsPerWarp];
  uint32_t e[kMaxRowsPerWarp / 8];
  uint32_t x[6];
};

__device__ __forceinline__ void load_strip(StripIn& o, const uint32_t* __restrict__ rec,
                                           const uint8_t* __restrict__ eplane,
                                           const uint16_t* __restrict__ x, const AmortGeom& g, int r0,
                                           int r1, int warp, int lane, int s) {
  const int u = s * kStrip + lane;
#pragma unroll
  for (int k = 0; k < kMaxRowsPerWarp / 8; ++k) o.e[k] = 0u;
#pragma unroll
  for (int i = 0; i < kMaxRowsPerWarp; ++i) {
    const int r = r0 + warp + kWarps * i;
    const bool ok = r < r1 && u < g.rec_pitch &&
                    SEEDLM_IN_BOUNDS(g_check_flag, (size_t)r * g.rec_pitch + u,
                                     (size_t)g.rows * g.rec_pitch);
    o.r[i] = ok ? ld_stream_u1(rec + (size_t)r * g.rec_pitch + u) : 0u;
    const bool eok = r < r1 && (u >> 1) < g.e_pitch &&
                     SEEDLM_IN_BOUNDS(g_check_flag, (size_t)r * g.e_pitch + (u >> 1),
                                      (size_t)g.rows * g.e_pitch);
    const uint32_t eb = eok ? (uint32_t)ld_stream_u8(eplane + (size_t)r * g.e_pitch + (u >> 1)) : 0u;
    o.e[i >> 3] |= ((eb >> (4 * (u & 1))) & 15u) << (4 * (i & 7));
  }
  // The table builder's column block is (thread % 32) = lane.
  const int col0 = u * 12;
#pragma unroll
  for (int k = 0; k < 6; ++k) {
    const int c = col0 + 2 * k;
    const uint32_t lo = c < g.cols ? x[c] : 0u;
    const uint32_t hi = c + 1 < g.cols ? x[c + 1] : 0u;
    o.x[k] = lo | (hi << 16);
  }
}

// X~_m for m = 8J .. 8J+7 (zero past 26): the first from its definition,
// the others by X~_m = 2 X~_{m-1} + 2^-15 x_m - 2 x_{m-16} (each x_c enters
// at m = c and leaves past m = c + 15).
template <int J>
__device__ __forceinline__ void x_tilde(const float (&xv)[12], float (&xt)[8]) {
  constexpr int m0 = 8 * J;
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < 12; ++c)
    if (m0 - c >= 0 && m0 - c <= 15) acc = fmaf(xv[c], __uint_as_float((uint32_t)(112 + m0 - c) << 23), acc);
  xt[0] = acc;
#pragma unroll
  for (int k = 1; k < 8; ++k) {
    const int m = m0 + k;
    float v = 2.f * xt[k - 1];
    if (m < 12) v = fmaf(xv[m < 12 ? m : 0], 0x1p-15f, v);
    if (m >= 16 && m - 16 < 12) v = fmaf(xv[m >= 16 && m - 16 < 12 ? m - 16 : 0], -2.f, v);
    xt[k] = m <= 26 ? v : 0.f;
  }
}

// Tables of strip s: thread t builds entries [64 q, 64 q + 64) of table j
// for column block l (t = l + 32 j + 128 q), from X~_{8j..8j+7} of that
// block: T_j[v] = A[v & 15] + B(v >> 4), A over bits 0..3, B over 4..7.
__device__ void build_tables(const StripIn& in, int is_bf16, const AmortGeom& g, int s) {
  const int t = threadIdx.x, l = t & 31, j = (t >> 5) & 3, q = t >> 7;
  float xv[12];
#pragma unroll
  for (int c = 0; c < 12; ++c) xv[c] = act_to_float((uint16_t)(in.x[c >> 1] >> (16 * (c & 1))), is_bf16);
  float xt[8];
  switch (j) {  // warp-uniform
    case 0: x_tilde<0>(xv, xt); break;
    case 1: x_tilde<1>(xv, xt); break;
    case 2: x_tilde<2>(xv, xt); break;
    default: x_tilde<3>(xv, xt); break;
  }
  // A[i] = sum of xt[k] over the set bits k of i, each from a smaller entry.
  float A[16];
  A[0] = 0.f;
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    const int low = i & -i;
    A[i] = A[i ^ low] + xt[low == 1 ? 0 : low == 2 ? 1 : low == 4 ? 2 : 3];
  }
  // This thread's high nibbles are 4q .. 4q + 3: bits 2, 3 of the high
  // nibble come from q.
  const float bq = ((q & 1) ? xt[6] : 0.f) + ((q & 2) ? xt[7] : 0.f);
  const uint32_t base = (j < 2 ? kT01 : kT23) + (uint32_t)(j & 1) * 128 + (uint32_t)l * 4;
#pragma unroll
  for (int hi = 0; hi < 4; ++hi) {
    const int vh = 4 * q + hi;  // v >> 4
    const float b = bq + ((hi & 1) ? xt[4] : 0.f) + ((hi & 2) ? xt[5] : 0.f);
#pragma unroll
    for (int lo = 0; lo < 16; ++lo) stsf(base + (uint32_t)((vh << 4) | lo) * 256, A[lo] + b);
  }
  if (j == 0 && q == 0) {
    float sx = 0.f;
#pragma unroll
    for (int c = 0; c < 12; ++c) sx += xv[c];
    stsf(kXsum + (uint32_t)l * 4, sx);
  }
}

// The lane's block of one row: its dot with the block's x, from the tables.
__device__ __forceinline__ float block_dot(uint32_t rec, uint32_t e4, float xsum, uint32_t lane4,
                                           uint32_t lane8) {
  // Stream bits 16..79 from the seed's bytes (rec bits 16..31).
  const uint2 a = ldsu2<kJump>(prmt<0x5524u>(rec, lane8));
  const uint2 b = ldsu2<kJump + 128>(prmt<0x5534u>(rec, lane8));
  const uint32_t mid = a.x ^ b.x, hi = a.y ^ b.y;   // stream bits 16..47, 48..79
  const uint32_t s0 = __funnelshift_r(rec, mid, 16);  // stream bits 0..31
  const uint32_t s1 = __funnelshift_r(mid, hi, 16);   // 32..63
  const uint32_t o0 = __funnelshift_r(s0, s1, 4);     // 4..35
  const uint32_t o1 = __funnelshift_r(mid, hi, 20);   // 36..67
  // S_p from the bytes at bits 12p, 12p + 8, 12p + 16, 12p + 24.
  const float S0 = ldsf<kT01>(row_addr<0>(s0, lane4)) + ldsf<kT01 + 128>(row_addr<1>(s0, lane4)) +
                   ldsf<kT23>(row_addr<2>(s0, lane4)) + ldsf<kT23 + 128>(row_addr<3>(s0, lane4));
  const float S1 = ldsf<kT01>(row_addr<1>(o0, lane4)) + ldsf<kT01 + 128>(row_addr<2>(o0, lane4)) +
                   ldsf<kT23>(row_addr<3>(o0, lane4)) + ldsf<kT23 + 128>(row_addr<0>(o1, lane4));
  const float S2 = ldsf<kT01>(row_addr<3>(s0, lane4)) + ldsf<kT01 + 128>(row_addr<0>(s1, lane4)) +
                   ldsf<kT23>(row_addr<1>(s1, lane4)) + ldsf<kT23 + 128>(row_addr<2>(s1, lane4));
  const float S3 = ldsf<kT01>(row_addr<0>(o1, lane4)) + ldsf<kT01 + 128>(row_addr<1>(o1, lane4)) +
                   ldsf<kT23>(row_addr<2>(o1, lane4)) + ldsf<kT23 + 128>(row_addr<3>(o1, lane4));
  // q_p (signed nibbles of rec bits 0..15) as floats, and their sum.
  const uint32_t sq = sext_nibble_bytes(prmt<0x5140u>(rec, rec >> 4) & 0x0f0f0f0fu);
  const float q0 = (float)(int8_t)(sq & 0xffu), q1 = (float)(int8_t)((sq >> 8) & 0xffu);
  const float q2 = (float)(int8_t)((sq >> 16) & 0xffu), q3 = (float)(int8_t)(sq >> 24);
  const float qs = (float)__dp4a((int)sq, 0x01010101, 0);
  float d = q0 * S0;
  d = fmaf(q1, S1, d);
  d = fmaf(q2, S2, d);
  d = fmaf(q3, S3, d);
  d = fmaf(-qs, xsum, d);
  return __uint_as_float(0x3f800000u - (e4 << 23)) * d;  // 2^-e
}

__global__ void __launch_bounds__(kWarps * 32, 1)
gemv_amort_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
                  const uint16_t* __restrict__ x, int is_bf16, float* __restrict__ y,
                  const __grid_constant__ AmortGeom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  // The next kernel in the stream may launch now; its CTAs take an SM when
  // this kernel's CTA there exits.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) != kBase) {
    if (threadIdx.x == 0) atomicOr(&g_amort_error, 1u);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lane4 = (uint32_t)lane << 2, lane8 = (uint32_t)(lane & 15) << 3;
  // Lane-replicated jump tables: row v (256 bytes) holds ext_lo(v) for lanes
  // 0..15, then ext_hi(v); thread i writes 16-byte piece i.
  for (int i = threadIdx.x; i < 4096; i += blockDim.x) {
    const int v = i >> 4, which = (i >> 3) & 1;
    const uint64_t e = which ? kStreamTables.hi[v] : kStreamTables.lo[v];
    const uint32_t a = kJump + (uint32_t)i * 16;
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %1, %2};" ::"r"(a), "r"((uint32_t)e),
                 "r"((uint32_t)(e >> 32))
                 : "memory");
  }
  // Records and x may be the previous kernel's output: read them only now.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int r0 = blockIdx.x * g.rows_per_cta;
  const int r1 = min(r0 + g.rows_per_cta, g.rows);
  float acc[kMaxRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kMaxRowsPerWarp; ++i) acc[i] = 0.f;
  for (int s = 0; s < g.strips; ++s) {
    // The strip's records are requested before the barrier, so that their
    // latency overlaps the wait for the other warps and the table build.
    StripIn in;
    load_strip(in, rec, eplane, x, g, r0, r1, warp, lane, s);
    __syncthreads();  // the previous strip's tables are no longer read
    build_tables(in, is_bf16, g, s);
    __syncthreads();  // this strip's tables are complete
    float xsum;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(xsum) : "r"(kXsum + lane4));
#pragma unroll
    for (int i = 0; i < kMaxRowsPerWarp; ++i) {
      if (r0 + warp + kWarps * i < r1) {
        const uint32_t e4 = (in.e[i >> 3] >> (4 * (i & 7))) & 15u;
        acc[i] += block_dot(in.r[i], e4, xsum, lane4, lane8);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxRowsPerWarp; ++i) {
    const int r = r0 + warp + kWarps * i;
    float v = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && r < r1 && SEEDLM_IN_BOUNDS(g_check_flag, r, g.rows)) y[r] = v;
  }
}

}  // namespace

bool gemv_amort_applies(const seedlm_format& f, const DeviceInfo& dev) {
  if (f.C != 12 || f.rows <= 0 || f.cols <= 0) return false;
  const int per_cta = (f.rows + dev.num_sms - 1) / dev.num_sms;
  return per_cta >= kMinRowsPerCta && per_cta <= kWarps * kMaxRowsPerWarp &&
         dev.max_smem_optin >= kSmemBytes;
}

int launch_gemv_amort(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                      const uint16_t* x, int is_bf16, float* y, cudaStream_t stream,
                      const DeviceInfo& dev) {
  if (!gemv_amort_applies(f, dev)) return SEEDLM_EUNSUPPORTED;
  AmortGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.rows_per_cta = (f.rows + dev.num_sms - 1) / dev.num_sms;
  g.strips = (f.nb + kStrip - 1) / kStrip;
  const int grid = (f.rows + g.rows_per_cta - 1) / g.rows_per_cta;
  const void* kern = (const void*)gemv_amort_kernel;
  int rc = allow_max_smem(kern, dev);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {(void*)&rec, (void*)&eplane, (void*)&x, (void*)&is_bf16, (void*)&y, (void*)&g};
  cudaError_t err = cudaLaunchKernelExC(&cfg, kern, args);
  if (err != cudaSuccess) return record_cuda_error(err);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

int read_and_clear_amort_error(unsigned int* out) {
  unsigned int v = 0, zero = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, g_amort_error, sizeof(v));
  if (err != cudaSuccess) return record_cuda_error(err);
  if (v) {
    err = cudaMemcpyToSymbol(g_amort_error, &zero, sizeof(zero));
    if (err != cudaSuccess) return record_cuda_error(err);
  }
  *out = v;
  return SEEDLM_OK;
}

}  // namespace seedlm
