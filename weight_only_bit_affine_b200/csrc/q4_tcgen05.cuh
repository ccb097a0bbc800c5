// q4_tcgen05.cuh -- 5th-generation tensor-core (tcgen05) and tensor-memory
// wrappers shared by the two tensor-core kernels, and the dequantization step
// that feeds them: w_hat = s*q + b split into two bf16 parts.
#pragma once

#include <cstdint>

#include "q4_device.cuh"

namespace q4 {

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Allocates `cols` tensor-memory columns (a power of two >= 32) for the CTA,
// writing the base address to *slot (shared memory); one whole warp calls it.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols) : "memory");
}

// Shared-memory matrix descriptor of a K-major operand with the 128-byte
// swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte
// offset), base 1024-byte aligned.  Adding 2 to the descriptor advances the
// start by 32 bytes (16 bf16 along K).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(16u >> 4) << 16;                // leading byte offset (unused with this swizzle)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;              // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                       // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                       // 128-byte swizzle
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: D fp32, A and B bf16,
// both K-major, M = 128, N = n (a multiple of 16, 16..256).
__host__ __device__ __forceinline__ uint32_t idesc_bf16_m128(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// D (tensor memory) [+]= A (tensor memory: 128 lanes x 8 columns of bf16
// pairs = K 16) x B (shared-memory descriptor).
__device__ __forceinline__ void tc_mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
      ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued before is complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 16 consecutive 32-bit columns of this thread's lane <- v (the warp's lane quarter).
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// 8 consecutive 32-bit columns of this thread's lane <- v.
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// W (8, 16 or 32) consecutive fp32 columns of this thread's lane into r;
// complete with tmem_wait_ld().
template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (W == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
  }
}

// ---- dequantization for the bf16 tensor-core operand ------------------------
//
// The MMA multiplies bf16 operands exactly, but w_hat = s*q + b generally
// needs more than bf16's 8 significant bits, and rounding it once would cost
// up to 2^-8 of |w_hat| per weight -- as much as the bf16 output rounding, and
// together more than the 4e-3 * sum|x w_hat| acceptance bound allows when the
// errors line up.  So each weight enters the MMA as two bf16 parts:
//
//   w32 = fp32(s*q + b)    (one fma: the product is exact, one rounding)
//   hi  = bf16(w32)        lo = bf16(w32 - hi)    (w32 - hi is exact in fp32)
//
// and two MMAs with the same activations accumulate x*hi + x*lo.  Then
// |w_hat - hi - lo| <= 2^-24 |w_hat| + 2^-8 |w32 - hi| <= ~2^-16 |w_hat|: the
// operand error is 256 times below the output rounding, with no cancellation
// anywhere (hi and lo have the sign of w_hat or are far smaller).

// bf16 -1.0: multiplies hi's bf16 halves in the exact subtraction below.
constexpr uint16_t kBf16MinusOne = 0xBF80u;

// q2: two exact codes as a bf16 pair (q_lo in bits 0..15, q_hi in 16..31);
// s: the group's bf16 scale bits; b: its bias as fp32; m1: kBf16MinusOne.
// Returns the pairs (hi_lo, hi_hi) and (lo_lo, lo_hi) in the same order.
__device__ __forceinline__ void split_hi_lo(uint32_t q2, uint16_t s, float b, uint16_t m1, uint32_t& hi,
                                            uint32_t& lo) {
  asm("{\n\t.reg .b16 ql, qh, hl, hh;\n\t.reg .f32 wl, wh, rl, rh;\n\t"
      "mov.b32 {ql, qh}, %2;\n\t"
      "fma.rn.f32.bf16 wl, ql, %3, %4;\n\t"
      "fma.rn.f32.bf16 wh, qh, %3, %4;\n\t"
      "cvt.rn.bf16x2.f32 %0, wh, wl;\n\t"
      "mov.b32 {hl, hh}, %0;\n\t"
      "fma.rn.f32.bf16 rl, hl, %5, wl;\n\t"
      "fma.rn.f32.bf16 rh, hh, %5, wh;\n\t"
      "cvt.rn.bf16x2.f32 %1, rh, rl;\n\t}"
      : "=r"(hi), "=r"(lo)
      : "r"(q2), "h"(s), "f"(b), "h"(m1));
}

}  // namespace q4
