// seedlm_device.cuh -- device building blocks shared by the SeedLM kernels.
//
// How a block is rebuilt here (the arithmetic is the pages' W_blk = U t; the
// organisation is this library's own, chosen for the sm_100 integer pipes):
//
// 1. The seed as a bit stream.  The register shifts right one place per step
//    and feeds a new bit in at the top, so state_k is bits [k, k+16) of one
//    bit stream b whose first 16 bits are the seed and whose later bits obey
//    b[m+16] = b[m] ^ b[m+2] ^ b[m+3] ^ b[m+5].  A block of C weights and P
//    columns needs stream bits [0, P*C + 15).  Bits 16.. depend linearly
//    (over GF(2)) on the seed, so ext(s) = ext(s & 0xff) ^ ext(s & 0xff00):
//    two 256-entry jump tables give the whole window with two shared-memory
//    reads and one xor, instead of P*C register steps.
//
// 2. Bytes instead of 16-bit states (C = 8).  With beta_j the j-th byte of the
//    32-bit window starting at bit c, state_{8p+c} = beta_p + 256 beta_{p+1},
//    so  sum_p q_p state_{8p+c} = sum_j kappa_j beta_j  with
//    kappa = (q0, q1 + 256 q0, q2 + 256 q1, 256 q2).  Two dp2a instructions
//    (16-bit coefficient x 8-bit byte, two products each) give the integer
//    weight from ONE funnel-shifted window per weight.  C = 12 has states 12
//    bits apart, so each state takes its own two bytes: coefficients
//    (q_p, 256 q_p) and four dp2a per weight.
//
// 3. Exact integer -> float with the scale folded in.  The block's integer
//    weight v = sum_p (state - 32768) q_p satisfies |v| < 2^20 and the weight
//    is v 2^-(15+e).  Adding v to the bit pattern of M_e = 1.5 * 2^(8-e)
//    (whose ulp is exactly 2^-(15+e)) and subtracting M_e in fp32 gives the
//    weight exactly, with the -32768 sum(q) offset folded into the same
//    integer start value.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace seedlm {

// ------------------------------------------------------------------ tables

// Stream bits 16..79 for a seed, by stepping the register 64 times.
constexpr uint64_t stream_ext(uint32_t seed) {
  uint32_t s = seed & 0xffffu;
  uint64_t out = 0;
  for (int k = 0; k < 64; ++k) {
    uint32_t bit = (s ^ (s >> 2) ^ (s >> 3) ^ (s >> 5)) & 1u;
    s = (s >> 1) | (bit << 15);
    out |= uint64_t(bit) << k;
  }
  return out;
}

struct StreamTables {
  uint64_t lo[256];  // ext(v)
  uint64_t hi[256];  // ext(v << 8)
};

constexpr StreamTables make_stream_tables() {
  StreamTables t{};
  for (uint32_t v = 0; v < 256; ++v) {
    t.lo[v] = stream_ext(v);
    t.hi[v] = stream_ext(v << 8);
  }
  return t;
}

// One copy per translation unit (4 KB), built at compile time.
static __device__ const StreamTables kStreamTables = make_stream_tables();

// ------------------------------------------------------------ PTX helpers

// prmt.b32 in its generic mode: each selector nibble picks one of the 8 bytes
// of {b, a}; bit 3 of the nibble replicates that byte's sign bit instead.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "n"(SEL));
  return d;
}

// d = c + a.s16[0] * b.u8[0] + a.s16[1] * b.u8[1]
__device__ __forceinline__ int32_t dp2a_lo_su(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// d = c + a.s16[0] * b.u8[2] + a.s16[1] * b.u8[3]
__device__ __forceinline__ int32_t dp2a_hi_su(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// d = c + a.s16[0] * b.s8[0] + a.s16[1] * b.s8[1]   (signed bytes)
__device__ __forceinline__ int32_t dp2a_lo_ss(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ int32_t dp2a_hi_ss(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Streaming 8-byte load that skips L1 allocation (records are read once).
__device__ __forceinline__ uint2 ld_stream_u2(const uint32_t* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_stream_u1(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint8_t ld_stream_u8(const uint8_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return (uint8_t)v;
}

// Prefetch of one line into L2, nothing returned to the thread.  It may be
// issued before griddepcontrol.wait even for data the previous kernel writes:
// the L2 is the point of coherence of the GPU's memory, so a write that lands
// after the prefetch updates the line in L2, and no copy nearer the SM is made.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// --------------------------------------------------------- block decoding

// Bit pattern of M_e = 1.5 * 2^(8-e) is 0x43C00000 - (e << 23).
constexpr uint32_t kMagicBits = 0x43C00000u;
constexpr uint32_t kNegMagicBits = 0xC3C00000u;

// Four signed bytes from four nibbles held one per byte (values 0..15):
// n >= 8 becomes n - 16, i.e. byte n | 0xF0.
__device__ __forceinline__ uint32_t sext_nibble_bytes(uint32_t v) {
  return v + (v & 0x08080808u) * 30u;
}

// Everything a C = 8, P = 3 block needs besides its windows.
struct BlockC8 {
  uint32_t lo;    // the record: seed in bits [16,32) = stream bits [0,16)
  uint32_t hi;    // stream bits [16,48)
  uint32_t a01;   // (kappa0, kappa1) as two s16
  uint32_t a23;   // (kappa2, kappa3) as two s16
  int32_t init;   // bits(M_e) - 32768 * (q0 + q1 + q2)
  uint32_t negm;  // bits(-M_e)
};

__device__ __forceinline__ BlockC8 decode_c8(uint32_t rec, const uint32_t* __restrict__ t_lo,
                                             const uint32_t* __restrict__ t_hi) {
  BlockC8 b;
  b.lo = rec;
  b.hi = t_lo[prmt<0x4442u>(rec, 0u)] ^ t_hi[rec >> 24];  // seed bytes 0 and 1
  // (q0, q1, q1, q2) as nibbles, one per byte, then sign-extended.
  uint32_t v = prmt<0x1440u>(rec, rec >> 4) & 0x0f0f0f0fu;
  uint32_t s = sext_nibble_bytes(v);
  int32_t k1 = dp2a_lo_ss(0x00010100u, s, 0);   // 256 q0 + q1
  int32_t k2 = dp2a_hi_ss(0x00010100u, s, 0);   // 256 q1 + q2
  b.a01 = prmt<0x5480u>(s, (uint32_t)k1);        // (q0, k1)
  b.a23 = ((uint32_t)k2 & 0xffffu) | (s & 0xff000000u);  // (k2, 256 q2)
  int32_t qsum = __dp4a((int)s, 0x01000101, 0);  // q0 + q1 + q2
  uint32_t e23 = (rec << 11) & 0x07800000u;      // e << 23
  b.init = (int32_t)(kMagicBits - e23) - qsum * 32768;
  b.negm = kNegMagicBits - e23;
  return b;
}

// Coefficient tables for C = 8 (built per CTA by fill_coef_tables_c8):
//   tq1[v], v = q0 | q1 << 4 (record byte 0):  (A01 = (q0, 256 q0 + q1), -32768 (q0 + q1))
//   tq2[v], v = q1 | q2 << 4 (record bits 4..11): (A23 = (256 q1 + q2, 256 q2), -32768 q2)
// with q the signed values of the nibbles.
__device__ __forceinline__ int32_t nibble_value(uint32_t n) { return (int32_t)(n & 15u) - (int32_t)((n & 8u) << 1); }

__device__ __forceinline__ uint32_t pack_s16(int32_t lo, int32_t hi) {
  return ((uint32_t)lo & 0xffffu) | ((uint32_t)hi << 16);
}

__device__ __forceinline__ void fill_coef_tables_c8(uint2* tq1, uint2* tq2, int tid, int nthreads) {
  for (int v = tid; v < 256; v += nthreads) {
    const int32_t a = nibble_value(v), b = nibble_value(v >> 4);
    tq1[v] = make_uint2(pack_s16(a, 256 * a + b), (uint32_t)(-32768 * (a + b)));
    tq2[v] = make_uint2(pack_s16(256 * a + b, 256 * b), (uint32_t)(-32768 * b));
  }
}

// decode_c8 with the coefficient part taken from the two tables above.
__device__ __forceinline__ BlockC8 decode_c8_tab(uint32_t rec, const uint32_t* __restrict__ t_lo,
                                                 const uint32_t* __restrict__ t_hi,
                                                 const uint2* __restrict__ tq1,
                                                 const uint2* __restrict__ tq2) {
  BlockC8 b;
  b.lo = rec;
  b.hi = t_lo[prmt<0x4442u>(rec, 0u)] ^ t_hi[rec >> 24];
  const uint2 c1 = tq1[rec & 0xffu];
  const uint2 c2 = tq2[(rec >> 4) & 0xffu];
  b.a01 = c1.x;
  b.a23 = c2.x;
  const uint32_t e23 = (rec << 11) & 0x07800000u;
  b.init = (int32_t)(kMagicBits - e23 + c1.y + c2.y);
  b.negm = kNegMagicBits - e23;
  return b;
}

// Integer weight c of a C = 8 block, biased by bits(M_e) (see 3. above).
template <int c>
__device__ __forceinline__ int32_t weight_bits_c8(const BlockC8& b) {
  uint32_t w = __funnelshift_r(b.lo, b.hi, 16 + c);  // stream bits [c, c+32)
  return dp2a_hi_su(b.a23, w, dp2a_lo_su(b.a01, w, b.init));
}

// Everything a C = 12, P = 4 block needs besides its windows.
struct BlockC12 {
  uint32_t lo;     // the record
  uint32_t mid;    // stream bits [16,48)
  uint32_t hi;     // stream bits [48,80)
  uint32_t a[4];   // (q_p, 256 q_p) as two s16
  int32_t init;
  uint32_t negm;
};

// The coefficient part of a C = 12 block: (q_p, 256 q_p) pairs, the integer
// start value and -M_e.  e4 is the block's exponent in bits [0,4).  SHIFT
// scales the weights by 2^SHIFT (added to the exponent of M_e).
template <int SHIFT = 0>
__device__ __forceinline__ void coef_c12(BlockC12& b, uint32_t rec, uint32_t e4) {
  uint32_t v = prmt<0x5140u>(rec, rec >> 4) & 0x0f0f0f0fu;  // (q0, q1, q2, q3)
  uint32_t s = sext_nibble_bytes(v);
  // (q_p, sign(q_p), 0x00, q_p): the zero byte is the sign of a byte of v.
  b.a[0] = prmt<0x0c80u>(s, v);
  b.a[1] = prmt<0x1c91u>(s, v);
  b.a[2] = prmt<0x2ca2u>(s, v);
  b.a[3] = prmt<0x3cb3u>(s, v);
  int32_t qsum = __dp4a((int)s, 0x01010101, 0);
  uint32_t e23 = (e4 & 15u) << 23;
  b.init = (int32_t)(kMagicBits + ((uint32_t)SHIFT << 23) - e23) - qsum * 32768;
  b.negm = kNegMagicBits + ((uint32_t)SHIFT << 23) - e23;
}

// e4 is the block's exponent in bits [0,4).
__device__ __forceinline__ BlockC12 decode_c12(uint32_t rec, uint32_t e4,
                                               const uint2* __restrict__ t_lo,
                                               const uint2* __restrict__ t_hi) {
  BlockC12 b;
  b.lo = rec;
  uint2 x0 = t_lo[(rec >> 16) & 0xffu];
  uint2 x1 = t_hi[rec >> 24];
  b.mid = x0.x ^ x1.x;
  b.hi = x0.y ^ x1.y;
  coef_c12(b, rec, e4);
  return b;
}

// 32-bit stream window starting at bit k (0 <= k < 48) of a C = 12 block.
template <int k>
__device__ __forceinline__ uint32_t window_c12(const BlockC12& b) {
  if constexpr (k < 16) return __funnelshift_r(b.lo, b.mid, 16 + k);
  else if constexpr (k == 16) return b.mid;
  else return __funnelshift_r(b.mid, b.hi, k - 16);
}

// Integer weight c of a C = 12 block, biased by bits(M_e).
//   state_c      = bytes 0,1 of window(c)
//   state_{c+12} = bytes 0,1 of window(c+12)
//   state_{c+24} = bytes 2,3 of window(c+8)
//   state_{c+36} = bytes 2,3 of window(c+20)
template <int c>
__device__ __forceinline__ int32_t weight_bits_c12(const BlockC12& b) {
  int32_t acc = dp2a_lo_su(b.a[0], window_c12<c>(b), b.init);
  acc = dp2a_lo_su(b.a[1], window_c12<c + 12>(b), acc);
  acc = dp2a_hi_su(b.a[2], window_c12<c + 8>(b), acc);
  return dp2a_hi_su(b.a[3], window_c12<c + 20>(b), acc);
}

__device__ __forceinline__ float weight_value(int32_t bits, uint32_t negm) {
  return __int_as_float(bits) + __uint_as_float(negm);
}

// Activation element -> float.
__device__ __forceinline__ float act_to_float(uint16_t bits, int is_bf16) {
  return is_bf16 ? __uint_as_float((uint32_t)bits << 16)
                 : __half2float(__ushort_as_half(bits));
}

}  // namespace seedlm
