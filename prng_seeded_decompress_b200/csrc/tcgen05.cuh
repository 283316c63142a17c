// tcgen05.cuh -- thin inline-PTX wrappers for the sm_100a tensor-core path:
// shared-memory matrix descriptors, tcgen05.mma (kind::f16, A from tensor
// memory, issued by one elected lane of a converged warp), TMEM allocation,
// loads and stores, bulk copies and mbarriers with bounded waits.
#pragma once

#include <stdint.h>

namespace seedlm {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor, K-major operand without swizzle.  The
// operand is stored as 8-row x 16-byte "core matrices"; `lbo` is the byte
// distance between core matrices adjacent along K, `sbo` between core
// matrices adjacent along M (or N).  Fields: start address >> 4 in bits
// [0,14), LBO >> 4 in [16,30), SBO >> 4 in [32,46), descriptor version 1 in
// [46,48), layout type 0 (no swizzle) in [61,64).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// Instruction descriptor for kind::f16: D fp32, A and B both fp16 (bf16 = 0)
// or both bf16 (bf16 = 1), K-major, M = 128, N = n (multiple of 16, <= 256).
__host__ __device__ constexpr uint32_t idesc_f16(int n, int bf16) {
  return (1u << 4)                        // D format: f32
         | ((uint32_t)bf16 << 7)          // A format: f16 / bf16
         | ((uint32_t)bf16 << 10)         // B format: f16 / bf16
         | ((uint32_t)(n >> 3) << 17)     // N >> 3
         | ((uint32_t)(128 >> 4) << 24);  // M >> 4
}

// kind::f16 MMA, K = 16, A from tensor memory (128 lanes = rows x 8 columns,
// each column two 16-bit elements, the lower K index in the low half), B from
// shared memory through its descriptor, D (fp32) in tensor memory.  Both
// this and the commit below are whole-warp forms: every lane of a converged
// warp calls them with the same (warp-uniform) operands and one elected lane
// issues the instruction, so the operands can stay in uniform registers.
__device__ __forceinline__ void mma_f16_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :
      : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u),
        "r"(0u), "r"(0u));
}
// Eight K = 16 steps of two pieces (16 MMAs) in one statement: piece pc of
// step k reads A at a0 + pc * pcols + 8 k and B at b_desc + 16 k (the
// descriptor's address field counts 16-byte units).  One elect for all.
__device__ __forceinline__ void mma_f16_ts_warp_8x2(uint32_t d_tmem, uint32_t a0, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b32 a<16>;\n\t.reg .b64 b<8>;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "add.u32 a1, %1, 64;\n\t add.u32 a2, %1, 8;\n\t add.u32 a3, %1, 72;\n\t"
      "add.u32 a4, %1, 16;\n\t add.u32 a5, %1, 80;\n\t add.u32 a6, %1, 24;\n\t add.u32 a7, %1, 88;\n\t"
      "add.u32 a8, %1, 32;\n\t add.u32 a9, %1, 96;\n\t add.u32 a10, %1, 40;\n\t add.u32 a11, %1, 104;\n\t"
      "add.u32 a12, %1, 48;\n\t add.u32 a13, %1, 112;\n\t add.u32 a14, %1, 56;\n\t add.u32 a15, %1, 120;\n\t"
      "add.u64 b1, %2, 16;\n\t add.u64 b2, %2, 32;\n\t add.u64 b3, %2, 48;\n\t add.u64 b4, %2, 64;\n\t"
      "add.u64 b5, %2, 80;\n\t add.u64 b6, %2, 96;\n\t add.u64 b7, %2, 112;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b3, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b3, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a8], b4, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a9], b4, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a10], b5, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a11], b5, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a12], b6, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a13], b6, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a14], b7, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a15], b7, %3, t;\n\t}\n"
      :
      : "r"(d_tmem), "r"(a0), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Six K = 16 steps of two pieces (12 MMAs) in one statement: piece pc of
// step k reads A at a0 + pc * 48 + 8 k and B at b_desc + 16 k.  One elect
// for all.
__device__ __forceinline__ void mma_f16_ts_warp_6x2(uint32_t d_tmem, uint32_t a0, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b32 a<12>;\n\t.reg .b64 b<6>;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "add.u32 a1, %1, 48;\n\t"
      "add.u32 a2, %1, 8;\n\t"
      "add.u32 a3, %1, 56;\n\t"
      "add.u32 a4, %1, 16;\n\t"
      "add.u32 a5, %1, 64;\n\t"
      "add.u32 a6, %1, 24;\n\t"
      "add.u32 a7, %1, 72;\n\t"
      "add.u32 a8, %1, 32;\n\t"
      "add.u32 a9, %1, 80;\n\t"
      "add.u32 a10, %1, 40;\n\t"
      "add.u32 a11, %1, 88;\n\t"
      "add.u64 b1, %2, 16;\n\t"
      "add.u64 b2, %2, 32;\n\t"
      "add.u64 b3, %2, 48;\n\t"
      "add.u64 b4, %2, 64;\n\t"
      "add.u64 b5, %2, 80;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b3, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b3, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a8], b4, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a9], b4, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a10], b5, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a11], b5, %3, t;\n\t}\n"
      :
      : "r"(d_tmem), "r"(a0), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Four K = 16 steps of two pieces (8 MMAs) in one statement: piece pc of
// step k reads A at a0 + pc * 32 + 8 k and B at b_desc + 16 k.  One elect
// for all.
__device__ __forceinline__ void mma_f16_ts_warp_4x2(uint32_t d_tmem, uint32_t a0, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b32 a<8>;\n\t.reg .b64 b<4>;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "add.u32 a1, %1, 32;\n\t"
      "add.u32 a2, %1, 8;\n\t"
      "add.u32 a3, %1, 40;\n\t"
      "add.u32 a4, %1, 16;\n\t"
      "add.u32 a5, %1, 48;\n\t"
      "add.u32 a6, %1, 24;\n\t"
      "add.u32 a7, %1, 56;\n\t"
      "add.u64 b1, %2, 16;\n\t"
      "add.u64 b2, %2, 32;\n\t"
      "add.u64 b3, %2, 48;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b3, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b3, %3, t;\n\t}\n"
      :
      : "r"(d_tmem), "r"(a0), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Three K = 16 steps of two pieces (6 MMAs) in one statement: piece pc of
// step k reads A at a0 + pc * 24 + 8 k and B at b_desc + 16 k.  One elect
// for all.
__device__ __forceinline__ void mma_f16_ts_warp_3x2(uint32_t d_tmem, uint32_t a0, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b32 a<6>;\n\t.reg .b64 b<3>;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "add.u32 a1, %1, 24;\n\t"
      "add.u32 a2, %1, 8;\n\t"
      "add.u32 a3, %1, 32;\n\t"
      "add.u32 a4, %1, 16;\n\t"
      "add.u32 a5, %1, 40;\n\t"
      "add.u64 b1, %2, 16;\n\t"
      "add.u64 b2, %2, 32;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b2, %3, t;\n\t}\n"
      :
      : "r"(d_tmem), "r"(a0), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit_warp(uint32_t mbar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n"
      :
      : "r"(mbar)
      : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// TMEM allocation (one full warp).  The allocated base address is written to
// shared memory at `slot`.
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :
               : "r"(slot), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               :
               : "r"(taddr), "r"(ncols)
               : "memory");
}

// 32 lanes x 16 columns of fp32 from TMEM (warp w reads lanes 32(w%4)..).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// The same load without the wait: the registers are valid only after
// tmem_wait_ld_tie on them.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// Waits for this thread's TMEM loads.  `r` passes through the wait, so no use
// of the loaded values can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld_tie(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// 32 lanes x 16 (or 8) 32-bit columns into TMEM; warp w writes lanes
// 32(w%4)..32(w%4)+31, thread i its own lane.  Complete with tmem_wait_st.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      :
      : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st2(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};"
               :
               : "r"(taddr), "r"(r[0]), "r"(r[1])
               : "memory");
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};"
               :
               : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
// Splits 16 K-consecutive weights w (fp32, exact multiples of 2^-24 below
// 2^11 in magnitude) into two fp16 pieces and stores them, two per 32-bit
// column with the lower K index in the low half: hi = w rounded toward zero
// to fp16 (its top 11 significant bits; all of w below fp16's normal range)
// into 8 columns at taddr_h, lo = w - hi (at most 9 bits, exact) into 8
// columns at taddr_l.  lo comes from one mixed-precision FMA per weight,
// (-1) * hi + w with hi in fp16.
__device__ __forceinline__ void tmem_st_f16_split_x8(uint32_t taddr_h, uint32_t taddr_l,
                                                     const float (&w)[16]) {
  asm volatile(
      "{\n\t.reg .b32 h<8>, l<8>;\n\t.reg .f16 g<16>, m;\n\t.reg .f32 d<16>;\n\t"
      "mov.b16 m, 0xBC00;\n\t"
      "cvt.rz.f16x2.f32 h0, %3, %2;\n\t"
      "mov.b32 {g0, g1}, h0;\n\t"
      "cvt.rz.f16x2.f32 h1, %5, %4;\n\t"
      "mov.b32 {g2, g3}, h1;\n\t"
      "cvt.rz.f16x2.f32 h2, %7, %6;\n\t"
      "mov.b32 {g4, g5}, h2;\n\t"
      "cvt.rz.f16x2.f32 h3, %9, %8;\n\t"
      "mov.b32 {g6, g7}, h3;\n\t"
      "cvt.rz.f16x2.f32 h4, %11, %10;\n\t"
      "mov.b32 {g8, g9}, h4;\n\t"
      "cvt.rz.f16x2.f32 h5, %13, %12;\n\t"
      "mov.b32 {g10, g11}, h5;\n\t"
      "cvt.rz.f16x2.f32 h6, %15, %14;\n\t"
      "mov.b32 {g12, g13}, h6;\n\t"
      "cvt.rz.f16x2.f32 h7, %17, %16;\n\t"
      "mov.b32 {g14, g15}, h7;\n\t"
      "fma.rn.f32.f16 d0, g0, m, %2;\n\t"
      "fma.rn.f32.f16 d1, g1, m, %3;\n\t"
      "fma.rn.f32.f16 d2, g2, m, %4;\n\t"
      "fma.rn.f32.f16 d3, g3, m, %5;\n\t"
      "fma.rn.f32.f16 d4, g4, m, %6;\n\t"
      "fma.rn.f32.f16 d5, g5, m, %7;\n\t"
      "fma.rn.f32.f16 d6, g6, m, %8;\n\t"
      "fma.rn.f32.f16 d7, g7, m, %9;\n\t"
      "fma.rn.f32.f16 d8, g8, m, %10;\n\t"
      "fma.rn.f32.f16 d9, g9, m, %11;\n\t"
      "fma.rn.f32.f16 d10, g10, m, %12;\n\t"
      "fma.rn.f32.f16 d11, g11, m, %13;\n\t"
      "fma.rn.f32.f16 d12, g12, m, %14;\n\t"
      "fma.rn.f32.f16 d13, g13, m, %15;\n\t"
      "fma.rn.f32.f16 d14, g14, m, %16;\n\t"
      "fma.rn.f32.f16 d15, g15, m, %17;\n\t"
      "cvt.rn.f16x2.f32 l0, d1, d0;\n\t"
      "cvt.rn.f16x2.f32 l1, d3, d2;\n\t"
      "cvt.rn.f16x2.f32 l2, d5, d4;\n\t"
      "cvt.rn.f16x2.f32 l3, d7, d6;\n\t"
      "cvt.rn.f16x2.f32 l4, d9, d8;\n\t"
      "cvt.rn.f16x2.f32 l5, d11, d10;\n\t"
      "cvt.rn.f16x2.f32 l6, d13, d12;\n\t"
      "cvt.rn.f16x2.f32 l7, d15, d14;\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {h0, h1, h2, h3, h4, h5, h6, h7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%1], {l0, l1, l2, l3, l4, l5, l6, l7};\n\t}\n"
      :
      : "r"(taddr_h), "r"(taddr_l), "f"(w[0]), "f"(w[1]), "f"(w[2]), "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]), "f"(w[7]), "f"(w[8]), "f"(w[9]), "f"(w[10]), "f"(w[11]), "f"(w[12]), "f"(w[13]), "f"(w[14]), "f"(w[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" : : "r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Plain arrival (release, CTA scope).
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" : : "r"(mbar) : "memory");
}
// Arrival that also expects `bytes` of asynchronous copies on this phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               :
               : "r"(mbar), "r"(bytes)
               : "memory");
}
// Plain (untiled, single-CTA) bulk copy of `bytes` from global memory to this
// CTA's shared memory; completion is counted on `mbar`.  Both addresses
// 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :
      : "r"(dst), "l"(src), "r"(bytes), "r"(mbar)
      : "memory");
}
// Barrier 1 over the first `n` threads of the CTA (n a multiple of 32).
__device__ __forceinline__ void named_sync(uint32_t n) {
  asm volatile("bar.sync 1, %0;" : : "r"(n) : "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits until the mbarrier's phase with the given parity has completed, for
// at most `limit_ns` nanoseconds.  Returns false if it gave up.
__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done)
      : "r"(mbar), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(mbar, parity)) return true;  // fast path: no timer read
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (done) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// try_wait that lets the hardware park the thread for up to `hint_ns`
// (woken early when the phase completes), so waiting warps do not take
// issue slots from working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t mbar, uint32_t parity, uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done)
      : "r"(mbar), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

// Both phases complete?  One round trip to the barrier unit for the two
// checks (the fast path of waiting on two barriers at once).
__device__ __forceinline__ bool mbar_try_wait2(uint32_t b1, uint32_t p1, uint32_t b2, uint32_t p2) {
  uint32_t d1, d2;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%2], %3;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 q, [%4], %5;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "selp.u32 %1, 1, 0, q;\n\t}\n"
      : "=r"(d1), "=r"(d2)
      : "r"(b1), "r"(p1), "r"(b2), "r"(p2)
      : "memory");
  return (d1 & d2) != 0;
}

// As mbar_wait, sharing one give-up flag across the CTA: once any wait has
// given up (and set *abort), every later wait returns false at once, so a
// broken hand-over costs one time-out, not one per wait.
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t mbar, uint32_t parity,
                                                   uint64_t limit_ns, volatile uint32_t* abort) {
  if (mbar_try_wait(mbar, parity)) return true;  // fast path: no timer read
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(mbar, parity, 20000u)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort = 1u;
      return false;
    }
  }
}

// As mbar_wait_or_abort but spinning on plain try_wait, with no suspend
// hint: for hand-overs every few hundred cycles, where a parked thread
// would wake too late.  The time limit is checked every 256 polls.
__device__ __forceinline__ bool mbar_spin_or_abort(uint32_t mbar, uint32_t parity,
                                                   uint64_t limit_ns, volatile uint32_t* abort) {
  if (mbar_try_wait(mbar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(mbar, parity)) return true;
    if ((n & 255u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort = 1u;
        return false;
      }
    }
  }
}

}  // namespace tc
}  // namespace seedlm
