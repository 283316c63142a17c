// gemm_tc.cu -- Y = X W^T for a small batch on the 5th-generation tensor
// cores (tcgen05), with W rebuilt on the fly.
//
// Where the batch makes the product a real contraction (several rows of X
// share every rebuilt weight), the reconstructed tiles feed tcgen05.mma
// (paperhub.cn review thread: the weights are rebuilt from s and t and then
// used to compute the activations).  The layout per CTA:
//
//   * D = W_tile (128 rows) x X^T (NB columns, NB = batch rounded up to 16)
//     accumulates in TMEM in fp32 (128 lanes x NB columns).
//   * Each K stage (64 columns for C = 8, 48 for C = 12, i.e. a whole number
//     of blocks) is built by all 512 threads: four threads per W row load the
//     row's records for the stage (one stage ahead, into registers), rebuild
//     the weights exactly in fp32 (see
//     seedlm_device.cuh) and split each into tf32 pieces hi + lo, both exact
//     (a weight has at most 21 significant bits; tf32 keeps 11).  X is
//     converted to fp32, which tf32 holds exactly for fp16 or bf16 inputs.
//     The operands are written in the K-major core-matrix layout (8 rows x
//     16 bytes per core matrix, no swizzle).
//   * One thread issues 2 x (stage K / 8) MMAs per stage (kind::tf32,
//     M = 128, N = NB) -- hi and lo pieces into the same accumulator -- and
//     commits them to the stage's mbarrier; the other threads go on building
//     the next stage.  A stage is rebuilt only after its MMAs have completed.
//   * Split-K: the columns are divided into `splits` ranges so that there are
//     about three CTAs per SM.  Each CTA writes its fp32 partial tile to the
//     caller's workspace; the last CTA of a row tile to arrive (atomic
//     counter) adds the partials in split order -- a fixed order, so every
//     call gives the same bits -- writes Y and resets the counter to zero.
//   * Every mbarrier wait is bounded; a wait that gives up raises the
//     library's device error flag, and TMEM is always released.
#include <cuda_runtime.h>

#include <mutex>

#include "seedlm_device.cuh"
#include "seedlm_internal.h"
#include "tcgen05.cuh"

namespace seedlm {

__device__ unsigned int g_tc_error = 0;

namespace {

constexpr int kTileM = 128;
constexpr int kThreads = 512;
constexpr uint64_t kWaitLimit = 2000000000ull;  // ns an mbarrier wait may take before giving up

template <int C>
struct TcCfg;
template <>
struct TcCfg<8> {
  static constexpr int KC = 64;  // columns per stage = 8 blocks
  static constexpr int STAGES = 2;
};
template <>
struct TcCfg<12> {
  static constexpr int KC = 48;  // 4 blocks
  static constexpr int STAGES = 3;
};

struct TcGeom {
  int rows, cols, nb, rec_pitch, e_pitch, M;
  int splits, chunks_per_split, nchunks, tiles;
  int x_vec;  // X rows are 8-byte aligned and cols % 4 == 0: load X 4 elements at a time
};

template <int C, int NB>
struct TcSmem {
  static constexpr int KC = TcCfg<C>::KC;
  static constexpr int STAGES = TcCfg<C>::STAGES;
  static constexpr int SBO = KC * 32;  // bytes between 8-row groups (KC/4 core matrices of 128 B)
  static constexpr int A_BYTES = kTileM * KC * 4;
  static constexpr int B_BYTES = NB * KC * 4;
  static constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
  static constexpr int TABLE_OFF = STAGES * STAGE_BYTES;
  static constexpr int TABLE_BYTES = (C == 8) ? 512 * 4 : 512 * 8;
  static constexpr int BAR_OFF = TABLE_OFF + TABLE_BYTES;  // STAGES mbarriers (8 B each)
  static constexpr int SLOT_OFF = BAR_OFF + 8 * STAGES;    // TMEM address, last-CTA flag
  static constexpr int TOTAL = SLOT_OFF + 16;
  static constexpr uint32_t TMEM_COLS = NB <= 32 ? 32 : 64;
};

// Byte offset of element (row, k) in a K-major core-matrix operand.
template <int SBO>
__device__ __forceinline__ uint32_t core_off(int row, int k4) {
  return (uint32_t)(row >> 3) * SBO + (uint32_t)k4 * 128u + (uint32_t)(row & 7) * 16u;
}

__device__ __forceinline__ void split_tf32(float w, float& hi, float& lo) {
  hi = __uint_as_float(__float_as_uint(w) & 0xFFFFE000u);
  lo = w - hi;  // exact; at most 10 significant bits, so exact in tf32 too
}

template <int C, int NB>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const uint32_t* __restrict__ rec, const uint8_t* __restrict__ eplane,
               const uint16_t* __restrict__ X, int is_bf16, float* __restrict__ Y,
               float* __restrict__ partial, unsigned int* __restrict__ counters, TcGeom g) {
  using L = TcSmem<C, NB>;
  constexpr int KC = L::KC, STAGES = L::STAGES, BLK = KC / C;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x / g.splits, split = blockIdx.x - tile * g.splits;
  const int r0 = tile * kTileM;
  const int c_begin = split * g.chunks_per_split;
  const int c_end = min(c_begin + g.chunks_per_split, g.nchunks);
  const int n_iter = c_end > c_begin ? c_end - c_begin : 0;

  uint32_t* t32 = reinterpret_cast<uint32_t*>(smem + L::TABLE_OFF);
  uint2* t64 = reinterpret_cast<uint2*>(smem + L::TABLE_OFF);
  for (int i = tid; i < 512; i += kThreads) {
    uint64_t v = i < 256 ? kStreamTables.lo[i] : kStreamTables.hi[i - 256];
    if constexpr (C == 8)
      t32[i] = (uint32_t)v;
    else
      t64[i] = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
  }
  const uint32_t bar0 = tc::smem_u32(smem + L::BAR_OFF);
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + L::SLOT_OFF);
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) tc::mbar_init(bar0 + 8 * s, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(tc::smem_u32(slot), L::TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = slot[0];
  const uint32_t idesc = tc::idesc_tf32(NB);
  bool ok = true;

  // Producer roles: four threads per W row, each rebuilding a quarter of the
  // row's blocks of the stage; the X slice is split over all threads.  The
  // next stage's records and X values are loaded before the current stage is
  // built.
  constexpr int BPT = BLK / 4;                                // blocks per thread
  constexpr int XCH = NB * (KC / 4);                          // 4-element X chunks per stage
  constexpr int XPT = (XCH + kThreads - 1) / kThreads;        // X chunks per thread
  // Warp w owns rows 8w..8w+7; lane l takes row 8w + (l & 7) and quarter
  // l >> 3, so the 8 lanes of a quarter-warp store to 8 different rows of a
  // core matrix (distinct banks).
  const int prow = 8 * warp + (lane & 7), pq = lane >> 3;
  const int gr = r0 + prow;
  const bool row_ok = gr < g.rows;

  struct Pref {
    uint32_t w[BPT];
    uint32_t e;
    uint2 x[XPT];
  };
  auto load_pref = [&](int chunk, Pref& p) {
    const int b_first = chunk * BLK + pq * BPT;
    const bool blk_ok = row_ok && b_first < g.nb;
    if constexpr (BPT == 2) {
      uint2 v = blk_ok ? ld_stream_u2(rec + (size_t)gr * g.rec_pitch + b_first) : make_uint2(0u, 0u);
      p.w[0] = v.x;
      p.w[1] = v.y;
    } else {
      p.w[0] = blk_ok ? __ldg(rec + (size_t)gr * g.rec_pitch + b_first) : 0u;
    }
    p.e = 0;
    if constexpr (C == 12)
      p.e = blk_ok ? (uint32_t)ld_stream_u8(eplane + (size_t)gr * g.e_pitch + (b_first >> 1)) : 0u;
#pragma unroll
    for (int k = 0; k < XPT; ++k) {
      const int i = tid + k * kThreads;
      const int k4 = i / NB, n = i - k4 * NB;  // n fastest: distinct banks when stored
      const int col = chunk * KC + 4 * k4;
      uint2 v = make_uint2(0u, 0u);
      if (i < XCH && n < g.M) {
        const uint16_t* src = X + (size_t)n * g.cols + col;
        if (g.x_vec) {
          if (col < g.cols) v = __ldg(reinterpret_cast<const uint2*>(src));
        } else {
          uint32_t h[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) h[u] = col + u < g.cols ? (uint32_t)__ldg(src + u) : 0u;
          v = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
        }
      }
      p.x[k] = v;
    }
  };

  // Build one stage from its prefetched records and X values.
  auto build_stage = [&](int it, const Pref& cur) {
    const int s = it % STAGES;
    const int use = it / STAGES;
    unsigned char* st = smem + s * L::STAGE_BYTES;
    if (use > 0) ok = tc::mbar_wait(bar0 + 8 * s, (use - 1) & 1, kWaitLimit) && ok;

    // ---- A: rebuilt weights, hi and lo tf32 pieces
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      float w[C];
      if constexpr (C == 8) {
        const BlockC8 blk = decode_c8(cur.w[i], t32, t32 + 256);
        const float nm = __uint_as_float(blk.negm);
        w[0] = __int_as_float(weight_bits_c8<0>(blk)) + nm;
        w[1] = __int_as_float(weight_bits_c8<1>(blk)) + nm;
        w[2] = __int_as_float(weight_bits_c8<2>(blk)) + nm;
        w[3] = __int_as_float(weight_bits_c8<3>(blk)) + nm;
        w[4] = __int_as_float(weight_bits_c8<4>(blk)) + nm;
        w[5] = __int_as_float(weight_bits_c8<5>(blk)) + nm;
        w[6] = __int_as_float(weight_bits_c8<6>(blk)) + nm;
        w[7] = __int_as_float(weight_bits_c8<7>(blk)) + nm;
      } else {
        const int b_first = (c_begin + it) * BLK + pq * BPT;
        const uint32_t e4 = (b_first & 1) ? (cur.e >> 4) : cur.e;
        const BlockC12 blk = decode_c12(cur.w[i], e4 & 15u, t64, t64 + 256);
        const float nm = __uint_as_float(blk.negm);
        w[0] = __int_as_float(weight_bits_c12<0>(blk)) + nm;
        w[1] = __int_as_float(weight_bits_c12<1>(blk)) + nm;
        w[2] = __int_as_float(weight_bits_c12<2>(blk)) + nm;
        w[3] = __int_as_float(weight_bits_c12<3>(blk)) + nm;
        w[4] = __int_as_float(weight_bits_c12<4>(blk)) + nm;
        w[5] = __int_as_float(weight_bits_c12<5>(blk)) + nm;
        w[6] = __int_as_float(weight_bits_c12<6>(blk)) + nm;
        w[7] = __int_as_float(weight_bits_c12<7>(blk)) + nm;
        w[8] = __int_as_float(weight_bits_c12<8>(blk)) + nm;
        w[9] = __int_as_float(weight_bits_c12<9>(blk)) + nm;
        w[10] = __int_as_float(weight_bits_c12<10>(blk)) + nm;
        w[11] = __int_as_float(weight_bits_c12<11>(blk)) + nm;
      }
      const int k4_0 = (pq * BPT + i) * (C / 4);
#pragma unroll
      for (int q = 0; q < C / 4; ++q) {
        float h[4], l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) split_tf32(w[4 * q + u], h[u], l[u]);
        const uint32_t off = core_off<L::SBO>(prow, k4_0 + q);
        *reinterpret_cast<float4*>(st + off) = make_float4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<float4*>(st + L::A_BYTES + off) = make_float4(l[0], l[1], l[2], l[3]);
      }
    }

    // ---- B: X[:, stage columns] as fp32 (exact in tf32), zero-padded
#pragma unroll
    for (int k = 0; k < XPT; ++k) {
      const int i = tid + k * kThreads;
      if (i < XCH) {
        const int k4 = i / NB, n = i - k4 * NB;
        const uint2 v = cur.x[k];
        const float4 f = make_float4(act_to_float((uint16_t)(v.x & 0xffffu), is_bf16),
                                     act_to_float((uint16_t)(v.x >> 16), is_bf16),
                                     act_to_float((uint16_t)(v.y & 0xffffu), is_bf16),
                                     act_to_float((uint16_t)(v.y >> 16), is_bf16));
        *reinterpret_cast<float4*>(st + 2 * L::A_BYTES + core_off<L::SBO>(n, k4)) = f;
      }
    }

    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t a_hi = tc::smem_u32(st), a_lo = a_hi + L::A_BYTES, bb = a_hi + 2 * L::A_BYTES;
#pragma unroll
      for (int kk = 0; kk < KC / 8; ++kk) {
        const uint64_t db = tc::smem_desc(bb + 256 * kk, 128, L::SBO);
        tc::mma_tf32(tmem, tc::smem_desc(a_hi + 256 * kk, 128, L::SBO), db, idesc,
                     (it > 0 || kk > 0) ? 1u : 0u);
        tc::mma_tf32(tmem, tc::smem_desc(a_lo + 256 * kk, 128, L::SBO), db, idesc, 1u);
      }
      tc::mma_commit(bar0 + 8 * s);
    }
  };

  // Record sets and X values are loaded two stages ahead of the one being
  // built (a ring of three register buffers, unrolled so they stay in
  // registers).
  Pref pf[3];
  if (n_iter > 0) load_pref(c_begin, pf[0]);
  if (n_iter > 1) load_pref(c_begin + 1, pf[1]);
  for (int it0 = 0; it0 < n_iter; it0 += 3) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int it = it0 + k;
      if (it < n_iter) {
        if (it + 2 < n_iter) load_pref(c_begin + it + 2, pf[(k + 2) % 3]);
        build_stage(it, pf[k]);
      }
    }
  }

  // ---- epilogue: wait for the last MMAs, read D, write Y or a partial
  float d[NB];
#pragma unroll
  for (int n = 0; n < NB; ++n) d[n] = 0.f;
  if (n_iter > 0) {
    const int s_last = (n_iter - 1) % STAGES, use_last = (n_iter - 1) / STAGES;
    ok = tc::mbar_wait(bar0 + 8 * s_last, use_last & 1, kWaitLimit) && ok;
    tc::fence_after_sync();
    if (warp < 4) {
#pragma unroll
      for (int n16 = 0; n16 < NB / 16; ++n16) {
        float v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + 16 * n16, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) d[16 * n16 + i] = v[i];
      }
    }
  }
  if (!ok) atomicOr(&g_tc_error, 1u);
  const int row = 32 * warp + lane;  // valid for warp < 4
  if (g.splits == 1) {
    if (warp < 4 && r0 + row < g.rows) {
#pragma unroll
      for (int n = 0; n < NB; ++n)
        if (n < g.M) Y[(size_t)n * g.rows + r0 + row] = d[n];
    }
  } else {
    float* mine = partial + ((size_t)(tile * g.splits + split) * NB) * kTileM;
    if (warp < 4) {
#pragma unroll
      for (int n = 0; n < NB; ++n) mine[n * kTileM + row] = d[n];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) slot[1] = (atomicAdd(&counters[tile], 1u) == (unsigned)(g.splits - 1)) ? 1u : 0u;
    __syncthreads();
    if (slot[1]) {
      __threadfence();
      const float* base = partial + ((size_t)tile * g.splits * NB) * kTileM;
      for (int i = tid; i < g.M * kTileM; i += kThreads) {
        const int n = i / kTileM, rr = i - n * kTileM;
        if (r0 + rr < g.rows) {
          float acc = 0.f;
          for (int sp = 0; sp < g.splits; ++sp) acc += base[((size_t)sp * NB + n) * kTileM + rr];
          Y[(size_t)n * g.rows + r0 + rr] = acc;
        }
      }
      if (tid == 0) counters[tile] = 0u;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, L::TMEM_COLS);
}

template <int C>
int tc_kc() {
  return TcCfg<C>::KC;
}

TcGeom make_tc_geom(const seedlm_format& f, int M, const DeviceInfo& dev) {
  TcGeom g;
  g.rows = f.rows;
  g.cols = f.cols;
  g.nb = f.nb;
  g.rec_pitch = f.rec_pitch;
  g.e_pitch = f.e_pitch;
  g.M = M;
  const int KC = f.C == 8 ? tc_kc<8>() : tc_kc<12>();
  g.nchunks = (f.cols + KC - 1) / KC;
  g.tiles = (f.rows + kTileM - 1) / kTileM;
  // About three CTAs per SM, each with at least 4 stages of work.
  int want = (3 * dev.num_sms + g.tiles - 1) / g.tiles;
  int cap = g.nchunks / 4 > 1 ? g.nchunks / 4 : 1;
  g.splits = want < 1 ? 1 : (want > cap ? cap : want);
  g.chunks_per_split = (g.nchunks + g.splits - 1) / g.splits;
  g.splits = (g.nchunks + g.chunks_per_split - 1) / g.chunks_per_split;
  g.x_vec = 0;
  return g;
}

template <int C, int NB>
int launch_tc(const TcGeom& g, const uint32_t* rec, const uint8_t* eplane, const uint16_t* X,
              int is_bf16, float* Y, float* partial, unsigned int* counters, cudaStream_t stream,
              const DeviceInfo& dev) {
  using L = TcSmem<C, NB>;
  if ((size_t)L::TOTAL > (size_t)dev.max_smem_optin) return SEEDLM_EUNSUPPORTED;
  int rc = allow_max_smem((const void*)gemm_tc_kernel<C, NB>, dev);
  if (rc) return rc;
  gemm_tc_kernel<C, NB><<<g.tiles * g.splits, kThreads, L::TOTAL, stream>>>(
      rec, eplane, X, is_bf16, Y, partial, counters, g);
  count_launch();
  return record_cuda_error(cudaGetLastError());
}

}  // namespace

int64_t gemm_tc_workspace_bytes(const seedlm_format& f, int M, const DeviceInfo& dev) {
  const TcGeom g = make_tc_geom(f, M, dev);
  if (g.splits <= 1) return 0;
  const int NB = (M + 15) / 16 * 16;
  const int64_t part = (int64_t)g.tiles * g.splits * NB * kTileM * 4;
  const int64_t cnt = ((int64_t)g.tiles * 4 + 255) / 256 * 256;
  return (part + 255) / 256 * 256 + cnt;
}

int launch_gemm_tc(const seedlm_format& f, const uint32_t* rec, const uint8_t* eplane,
                   const uint16_t* X, int is_bf16, int M, float* Y, void* workspace,
                   int64_t workspace_bytes, cudaStream_t stream, const DeviceInfo& dev) {
  TcGeom g = make_tc_geom(f, M, dev);
  g.x_vec = (f.cols % 4 == 0 && (reinterpret_cast<uintptr_t>(X) & 7u) == 0) ? 1 : 0;
  const int64_t need = gemm_tc_workspace_bytes(f, M, dev);
  if (workspace_bytes < need) return SEEDLM_EINVAL;
  float* partial = nullptr;
  unsigned int* counters = nullptr;
  if (need > 0) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SEEDLM_EINVAL;
    const int NB = (M + 15) / 16 * 16;
    const int64_t part = ((int64_t)g.tiles * g.splits * NB * kTileM * 4 + 255) / 256 * 256;
    partial = static_cast<float*>(workspace);
    counters = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + part);
  }
  const int NB = (M + 15) / 16 * 16;
  if (f.C == 8) {
    switch (NB) {
      case 16: return launch_tc<8, 16>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
      case 32: return launch_tc<8, 32>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
      case 48: return launch_tc<8, 48>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
      default: return launch_tc<8, 64>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
    }
  }
  switch (NB) {
    case 16: return launch_tc<12, 16>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
    case 32: return launch_tc<12, 32>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
    case 48: return launch_tc<12, 48>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
    default: return launch_tc<12, 64>(g, rec, eplane, X, is_bf16, Y, partial, counters, stream, dev);
  }
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
// For callers that cannot allocate device memory themselves, the split-K
// partial tiles and the per-tile counters of the tensor-core GEMM live in one
// array that the library owns for the life of the process.

constexpr int64_t kNoAllocPartialBytes = 16ll << 20;  // split-K partial tiles
constexpr int64_t kNoAllocCounterBytes = 64ll << 10;  // one uint32 per 128-row tile
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[kNoAllocPartialBytes + kNoAllocCounterBytes];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the name is only a host-side stand-in for it).
int noalloc_scratch(const DeviceInfo& dev, unsigned char** out) {
  if (dev.device < 0 || dev.device >= 64) return SEEDLM_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev.device]) {
    void* p = nullptr;
    cudaError_t err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return record_cuda_error(err);
    if (!p) return SEEDLM_ECUDA;
    g_noalloc_addr[dev.device] = p;
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
  if (!fmt) return SEEDLM_EINVAL;
  const bool c8 = fmt->C == 8 && fmt->P == 3 && fmt->K == 16;
  const bool c12 = fmt->C == 12 && fmt->P == 4 && fmt->K == 16;
  if (!c8 && !c12) return SEEDLM_EUNSUPPORTED;
  if (fmt->rows < 0 || fmt->cols < 0 || fmt->nb != (fmt->cols + fmt->C - 1) / fmt->C ||
      fmt->rec_pitch < fmt->nb || fmt->rec_pitch % 4 != 0 ||
      (c12 && fmt->e_pitch < (fmt->nb + 1) / 2))
    return SEEDLM_EINVAL;
  if (x_dtype != SEEDLM_F16 && x_dtype != SEEDLM_BF16) return SEEDLM_EINVAL;
  if (M < 1 || M > 64) return SEEDLM_EINVAL;
  if (fmt->rows == 0) return SEEDLM_OK;
  if (fmt->nb > 0 && (!rec || (reinterpret_cast<uintptr_t>(rec) & 15u))) return SEEDLM_EINVAL;
  if (fmt->nb > 0 && c12 && !eplane) return SEEDLM_EINVAL;
  if (!Y || (reinterpret_cast<uintptr_t>(Y) & 3u)) return SEEDLM_EINVAL;
  if (fmt->cols > 0 && (!X || (reinterpret_cast<uintptr_t>(X) & 1u))) return SEEDLM_EINVAL;
  DeviceInfo dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  if (fmt->cols == 0)
    return record_cuda_error(cudaMemsetAsync(Y, 0, (size_t)M * fmt->rows * sizeof(float), st));
  const uint16_t* Xh = static_cast<const uint16_t*>(X);
  const int is_bf16 = x_dtype == SEEDLM_BF16;
  if (M == 1) return launch_gemv(*fmt, rec, eplane, Xh, is_bf16, Y, st, dev);

  TcGeom g = make_tc_geom(*fmt, M, dev);
  g.x_vec = (fmt->cols % 4 == 0 && (reinterpret_cast<uintptr_t>(X) & 7u) == 0) ? 1 : 0;
  const int NB = (M + 15) / 16 * 16;
  const int64_t part_bytes =
      g.splits > 1 ? (int64_t)g.tiles * g.splits * NB * kTileM * (int64_t)sizeof(float) : 0;
  const int64_t cnt_bytes = g.splits > 1 ? (int64_t)g.tiles * 4 : 0;
  if (part_bytes > kNoAllocPartialBytes || cnt_bytes > kNoAllocCounterBytes)
    return SEEDLM_EUNSUPPORTED;  // needs more scratch than the library holds
  float* partial = nullptr;
  unsigned int* counters = nullptr;
  if (g.splits > 1) {
    unsigned char* base = nullptr;
    if ((rc = noalloc_scratch(dev, &base))) return rc;
    partial = reinterpret_cast<float*>(base);
    counters = reinterpret_cast<unsigned int*>(base + kNoAllocPartialBytes);
    // The counters must start at zero; the last call may have left them in
    // any state if it failed part-way.
    if ((rc = record_cuda_error(cudaMemsetAsync(counters, 0, (size_t)cnt_bytes, st)))) return rc;
  }
  if (fmt->C == 8) {
    switch (NB) {
      case 16: return launch_tc<8, 16>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
      case 32: return launch_tc<8, 32>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
      case 48: return launch_tc<8, 48>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
      default: return launch_tc<8, 64>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
    }
  }
  switch (NB) {
    case 16: return launch_tc<12, 16>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
    case 32: return launch_tc<12, 32>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
    case 48: return launch_tc<12, 48>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
    default: return launch_tc<12, 64>(g, rec, eplane, Xh, is_bf16, Y, partial, counters, st, dev);
  }
}
