// rep_tables.cuh -- lane-replicated decode tables at fixed shared addresses,
// shared by the GEMV and the tensor-core GEMM.
//
// Every decode table (the stream jump tables, and for C = 8 the coefficient
// tables) is stored once per lane, in rows of 256 bytes: row v holds entry v
// for each lane side by side (4-byte entries: lanes 0..31; 8-byte entries:
// lanes 0..15, one half-warp at a time).  Lane l always reads its own bank
// (bank pair), whatever index it looks up: one shared-memory wavefront per
// lookup instead of about 3.2 for random indices into a single copy.
//
// The rows start at fixed shared addresses, so the address of (row v, lane l)
// is (v << 8) | lane_offset: one prmt moves the record's index byte next to
// the lane's offset byte, and the table base rides in the load's immediate
// offset.  A kernel using them must find its dynamic shared allocation at
// shared address kSmemBase (it checks at entry).
//
//   C = 8:  [0x10000, 0x20000)  jump rows   (ext_lo(v) lanes 0..31, ext_hi(v) lanes 0..31)
//           [0x20000, 0x30000)  coef rows   (tq1(v) lanes 0..15, tq2(v) lanes 0..15)
//   C = 12: [0x20000, 0x30000)  jump rows   (8-byte ext_lo(v) lanes 0..15, then ext_hi(v))
//
// SHIFT scales every rebuilt weight by 2^SHIFT exactly: it is added to the
// exponent of the magic number M_e (seedlm_device.cuh), whose ulp then is
// 2^(SHIFT - 15 - e).
#pragma once

#include "seedlm_device.cuh"

namespace seedlm {
namespace rep {

constexpr uint32_t kSmemBase = 1024;  // shared address of the dynamic allocation
constexpr uint32_t kJump8 = 0x10000;
constexpr uint32_t kCoef8 = 0x20000;
constexpr uint32_t kJump12 = 0x20000;
constexpr uint32_t kEnd = 0x30000;  // first shared address past the tables

// Lowest table address for a format: shared memory below it (from kSmemBase)
// and from kEnd on is free for the kernel.
template <int C>
__host__ __device__ constexpr uint32_t tables_begin() { return C == 8 ? kJump8 : kJump12; }

template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
  return v;
}

template <uint32_t OFF>
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
  return v;
}

// Fills the rows; smem is the dynamic allocation (at kSmemBase), shared by
// `nthreads` threads of which this is `tid`.  Coefficient entries, with q
// the signed nibble values:
//   tq1(v), v = q0 | q1 << 4: (kappa0, kappa1) = (q0, 256 q0 + q1) and
//           bits(1.5 * 2^(8 + SHIFT)) - 32768 (q0 + q1)
//   tq2(v), v = q1 | q2 << 4: (kappa2, kappa3) = (256 q1 + q2, 256 q2) and
//           -32768 q2
// so that a block's integer start value is tq1.y + tq2.y - (e << 23).
template <int C, int SHIFT>
__device__ void fill_rep_tables(unsigned char* smem, int tid, int nthreads) {
  // 16-byte piece i = 16 v + 8 which + k of the tables: piece k of half-row
  // (v, which), which = 0 the low 128 bytes of row v, 1 the high ones.  Eight
  // consecutive threads write one contiguous half-row, so every quarter-warp
  // store covers the 32 banks once (one thread per half-row would put all 32
  // lanes of a warp 256 bytes apart, on the same four banks).
  uint4* jr = reinterpret_cast<uint4*>(smem + (tables_begin<C>() - kSmemBase));
#pragma unroll 4
  for (int i = tid; i < 4096; i += nthreads) {
    const int v = i >> 4, which = (i >> 3) & 1;
    const uint64_t e = which ? kStreamTables.hi[v] : kStreamTables.lo[v];
    const uint32_t lo = (uint32_t)e, hi = (uint32_t)(e >> 32);
    jr[i] = (C == 8) ? make_uint4(lo, lo, lo, lo) : make_uint4(lo, hi, lo, hi);
  }
  if constexpr (C == 8) {
    constexpr uint32_t kMagic = kMagicBits + ((uint32_t)SHIFT << 23);
    uint4* cr = reinterpret_cast<uint4*>(smem + (kCoef8 - kSmemBase));
#pragma unroll 4
    for (int i = tid; i < 4096; i += nthreads) {
      const int v = i >> 4, which = (i >> 3) & 1;
      const int32_t a = nibble_value(v), b = nibble_value(v >> 4);
      const uint2 e = which == 0
                          ? make_uint2(pack_s16(a, 256 * a + b), kMagic - (uint32_t)(32768 * (a + b)))
                          : make_uint2(pack_s16(256 * a + b, 256 * b), (uint32_t)(-32768 * b));
      cr[i] = make_uint4(e.x, e.y, e.x, e.y);
    }
  }
}

// C = 8 decode.  The record's bytes 2 and 3 are the seed's low and high
// bytes, byte 0 is q0 | q1 << 4 and bits 4..11 are q1 | q2 << 4.  lane4 =
// 4 * lane, lane8 = 8 * (lane % 16).
template <int SHIFT>
__device__ __forceinline__ BlockC8 decode_c8_rep(uint32_t rec, uint32_t lane4, uint32_t lane8) {
  BlockC8 b;
  b.lo = rec;
  b.hi = lds32<kJump8>(prmt<0x5524u>(rec, lane4)) ^ lds32<kJump8 + 128>(prmt<0x5534u>(rec, lane4));
  const uint2 c1 = lds64<kCoef8>(prmt<0x5504u>(rec, lane8));
  const uint2 c2 = lds64<kCoef8 + 128>(prmt<0x5514u>(rec << 4, lane8));
  b.a01 = c1.x;
  b.a23 = c2.x;
  const uint32_t e23 = (rec << 11) & 0x07800000u;  // e << 23
  b.init = (int32_t)(c1.y + c2.y - e23);
  b.negm = kNegMagicBits + ((uint32_t)SHIFT << 23) - e23;
  return b;
}

// C = 12 decode: stream windows from the 8-byte jump rows, the coefficients
// computed from the record's nibbles.  e4 is the block's exponent in bits [0,4).
template <int SHIFT>
__device__ __forceinline__ BlockC12 decode_c12_rep(uint32_t rec, uint32_t e4, uint32_t lane8) {
  BlockC12 b;
  b.lo = rec;
  const uint2 x0 = lds64<kJump12>(prmt<0x5524u>(rec, lane8));
  const uint2 x1 = lds64<kJump12 + 128>(prmt<0x5534u>(rec, lane8));
  b.mid = x0.x ^ x1.x;
  b.hi = x0.y ^ x1.y;
  coef_c12<SHIFT>(b, rec, e4);
  return b;
}

}  // namespace rep
}  // namespace seedlm
