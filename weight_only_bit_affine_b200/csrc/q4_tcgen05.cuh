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

// True in exactly one lane of the (converged) warp, the same lane every time.
// The MMA-issuing loops run on a whole warp, so their descriptors and
// tensor-memory addresses are warp-uniform values, and only the issue itself
// (an MMA, a commit) is made by the elected lane: issued from a lone lane
// (lane == 0), every operand would first be moved to the uniform datapath.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(pred));
  return pred != 0;
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
//
// Instruction count per pair of weights: the codes become exact fp32 values
// in place (unpack_codes_f32: a LOP3 per code, a packed add per pair), w32 is
// one packed fp32 fma (fma.rn.f32x2), hi one conversion, the remainder one
// packed subtraction of hi widened back to fp32 (a shift and an AND), lo one
// conversion.

// {v, v} as the 64-bit operand of the packed fp32 instructions.
__device__ __forceinline__ uint64_t f32x2_splat(float v) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
  return r;
}

// One pair (q0, q1) of exact codes in fp32 -> the bf16 pairs hi = (hi0, hi1)
// and lo = (lo0, lo1) of s*q + b (element 0 in bits 0..15); s2 = {s, s}, b2 =
// {b, b} from f32x2_splat.
__device__ __forceinline__ void split_pair(float q0, float q1, uint64_t s2, uint64_t b2, uint32_t& hi,
                                           uint32_t& lo) {
  asm("{\n\t.reg .b64 rq, rw, rh, rr;\n\t.reg .f32 w0, w1, r0, r1;\n\t.reg .b32 t0, t1;\n\t"
      "mov.b64 rq, {%2, %3};\n\t"
      "fma.rn.f32x2 rw, rq, %4, %5;\n\t"
      "mov.b64 {w0, w1}, rw;\n\t"
      "cvt.rn.bf16x2.f32 %0, w1, w0;\n\t"
      "shl.b32 t0, %0, 16;\n\t"
      "and.b32 t1, %0, 0xFFFF0000;\n\t"
      "mov.b64 rh, {t0, t1};\n\t"
      "sub.rn.f32x2 rr, rw, rh;\n\t"
      "mov.b64 {r0, r1}, rr;\n\t"
      "cvt.rn.bf16x2.f32 %1, r1, r0;\n\t}"
      : "=r"(hi), "=r"(lo)
      : "f"(q0), "f"(q1), "l"(s2), "l"(b2));
}

// One packed word (codes of eight consecutive k, q_j in bits 4j..4j+3) ->
// four hi and four lo bf16 pairs, pair i = (k 2i, k 2i+1).  Each code becomes
// an exact fp32 in place: masked into the significand of 2^(23-p), where its
// lowest bit p weighs 1, then the offsets 2^(23-p) removed by one packed add
// per pair (codes 5..7 are shifted down by 12 bits first).
__device__ __forceinline__ void dequant_word_hilo(uint32_t w, uint64_t s2, uint64_t b2, uint32_t* hi, uint32_t* lo) {
  const uint32_t ws = w >> 12;
  float q0, q1;
  q0 = __uint_as_float((w & 0x0000000Fu) | 0x4B000000u);   // 2^23 + q0
  q1 = __uint_as_float((w & 0x000000F0u) | 0x49000000u);   // 2^19 + q1
  fadd2(q0, q1, -8388608.f, -524288.f);
  split_pair(q0, q1, s2, b2, hi[0], lo[0]);
  q0 = __uint_as_float((w & 0x00000F00u) | 0x47000000u);   // 2^15 + q2
  q1 = __uint_as_float((w & 0x0000F000u) | 0x45000000u);   // 2^11 + q3
  fadd2(q0, q1, -32768.f, -2048.f);
  split_pair(q0, q1, s2, b2, hi[1], lo[1]);
  q0 = __uint_as_float((w & 0x000F0000u) | 0x43000000u);   // 2^7 + q4
  q1 = __uint_as_float((ws & 0x00000F00u) | 0x47000000u);  // 2^15 + q5
  fadd2(q0, q1, -128.f, -32768.f);
  split_pair(q0, q1, s2, b2, hi[2], lo[2]);
  q0 = __uint_as_float((ws & 0x0000F000u) | 0x45000000u);  // 2^11 + q6
  q1 = __uint_as_float((ws & 0x000F0000u) | 0x43000000u);  // 2^7 + q7
  fadd2(q0, q1, -2048.f, -128.f);
  split_pair(q0, q1, s2, b2, hi[3], lo[3]);
}

}  // namespace q4
