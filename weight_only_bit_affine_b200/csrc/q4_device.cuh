// q4_device.cuh -- device-side helpers shared by the libq4 kernels:
// PTX wrappers for mbarriers, 1-D bulk (TMA) copies, L2 prefetch,
// programmatic dependent launch, bounded waits, and bf16 bit tricks.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "q4_internal.h"

namespace q4 {

// Set (never cleared by kernels) when a bounded wait gives up.  Each
// translation unit has its own copy; the host reads and clears them through
// q4_device_status().
enum : unsigned int { kFlagWaitTimeout = 1u };
static __device__ unsigned int g_device_flags = 0;

// Host side: read (and optionally clear) this translation unit's flag word.
static inline cudaError_t tu_device_flags(unsigned int* flags, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_device_flags, sizeof(unsigned int));
  if (e == cudaSuccess && clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_device_flags, &zero, sizeof(unsigned int));
  }
  return e;
}

// A wait gives up after this many nanoseconds of %globaltimer (1 s): far
// beyond any legitimate wait in these kernels.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- programmatic dependent launch --------------------------------------
// Let the next kernel in the stream start its prologue now.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Block until every kernel this one depends on has completed and its writes
// are visible.  A no-op when the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait_predecessors() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// As mbar_try_wait, but a thread whose phase is not complete is suspended
// (not spinning, so it takes no issue slots from working warps) until the
// phase completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
  return ok != 0;
}
#ifndef Q4_WAIT_SLEEP_NS
#define Q4_WAIT_SLEEP_NS 20000u
#endif
// Wait for the phase with the given parity to complete.  Returns false (and
// raises the device flag) if it has not completed within kWaitLimitNs.
// kSleep selects the suspend-hinted form (for waits that are usually long,
// so the waiting warp leaves its issue slots to the others).
template <bool kSleep = true>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 16; ++i) {
      if constexpr (kSleep) {
        if (mbar_try_wait_sleep(bar, parity, Q4_WAIT_SLEEP_NS)) return true;
      } else {
        if (mbar_try_wait(bar, parity)) return true;
      }
    }
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_device_flags, kFlagWaitTimeout);
      return false;
    }
  }
}

// As mbar_wait, but between polls the thread sleeps about kNs nanoseconds
// (nanosleep): a polling warp takes no issue slots and no ALU cycles from
// the warps that do the work on its SM sub-partition while it waits.
template <unsigned kNs>
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 8; ++i) {
      __nanosleep(kNs);
      if (mbar_try_wait(bar, parity)) return true;
    }
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_device_flags, kFlagWaitTimeout);
      return false;
    }
  }
}

// ---- grid-wide stage counters (persistent chain launches) ------------------
// One CTA thread announces that the CTA finished a stage: a GPU-scope fence
// (cumulative: it orders the writes of the CTA's other threads that this
// thread has synchronized with, through an mbarrier, before the add) and a
// release add.
__device__ __forceinline__ void grid_arrive(unsigned int* counter) {
  asm volatile("fence.acq_rel.gpu;\n\tred.release.gpu.global.add.u32 [%0], 1;" ::"l"(counter) : "memory");
}

// Waits until *counter >= target (acquire loads at GPU scope, a short sleep
// between them).  Returns false (and raises the device flag) after
// kWaitLimitNs.
__device__ __forceinline__ bool grid_wait(const unsigned int* counter, unsigned int target) {
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= target) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_device_flags, kFlagWaitTimeout);
      return false;
    }
    __nanosleep(32);
  }
}

// ---- bulk (non-tensor TMA) copies and prefetch ----------------------------
// Global -> shared, completion counted in bytes on `bar`.  dst, src 16-byte
// aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// Hint: bring [src, src+bytes) into L2.  No effect on memory semantics.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---- named barriers ---------------------------------------------------------
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- bf16 helpers -------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t float_to_bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// ---- output epilogues (kEpi* in q4_internal.h) ----------------------------------
// silu(z) = z * sigmoid(z) = z / (1 + e^-z); e^-z overflows to +inf for very
// negative z, giving the correct limit -0.
__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + expf(-z)); }

__device__ __forceinline__ uint16_t epilogue_bf16(float acc, int epi, const uint16_t* r, int64_t idx) {
  if (epi == kEpiResidual) return float_to_bf16_bits(acc + bf16_bits_to_float(r[idx]));
  return float_to_bf16_bits(acc);
}

// Four codes of a packed word -> bf16x2 (128 + q[t], 128 + q[t + 4]).  0x4300
// is bf16 128.0, whose last significand bit weighs 1, so OR-ing a nibble into
// the low mantissa bits gives exactly 128 + q.
__device__ __forceinline__ uint32_t nibbles_to_bf16x2_plus128(uint32_t word, int t) {
  return ((word >> (4 * t)) & 0x000F000Fu) | 0x43004300u;
}

// d = a * b + c with a, b bf16 (exact product) and c, d fp32: one rounding.
// Two lanes of bf16x2 operands into two fp32 accumulators.
__device__ __forceinline__ void fma_bf16x2_f32(float& c0, float& c1, uint32_t a2, uint32_t b2) {
  asm("{ .reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %1, ah, bh, %1; }"
      : "+f"(c0), "+f"(c1) : "r"(a2), "r"(b2));
}

// One packed word (codes q0..q7 of eight consecutive inputs) against x:
//   c0 += sum_{t<4} x[t] * (128 + q[t]),   c1 += sum_{t<4} x[t+4] * (128 + q[t+4])
// x arrives as four bf16x2 registers xp[t] = (x[t], x[t+4]).  Each
// "128 + q" pair is one LOP3 on the word shifted by 4t (0x4300 = bf16 128.0,
// whose last significand bit weighs 1), and fma.rn.f32.bf16 multiplies the
// bf16 halves exactly and accumulates in fp32 with one rounding.  Written as
// one PTX block so the 16-bit halves are used in place (no extraction moves).
// The LOP3 constants (mask 0x000F000F, magic 0x43004300) come in registers
// that the caller holds across its loop (see q4_lop3_constants): given as two
// immediates, each LOP3 would rebuild one of them first.
__device__ __forceinline__ void q4_lop3_constants(uint32_t& mask, uint32_t& magic) {
  mask = 0x000F000Fu;
  magic = 0x43004300u;
  asm volatile("" : "+r"(mask), "+r"(magic));  // opaque: kept in registers, not rebuilt per use
}

__device__ __forceinline__ void word_dot_bf16(uint32_t w, uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                                              float& c0, float& c1, uint32_t mask, uint32_t magic) {
  asm("{\n\t.reg .b32 s1, s2, s3, v0, v1, v2, v3;\n\t"
      ".reg .b16 l0, h0, l1, h1, l2, h2, l3, h3, xl0, xh0, xl1, xh1, xl2, xh2, xl3, xh3;\n\t"
      "shr.b32 s1, %2, 4;\n\t"
      "shr.b32 s2, %2, 8;\n\t"
      "shr.b32 s3, %2, 12;\n\t"
      "lop3.b32 v0, %2, %7, %8, 0xEA;\n\t"
      "lop3.b32 v1, s1, %7, %8, 0xEA;\n\t"
      "lop3.b32 v2, s2, %7, %8, 0xEA;\n\t"
      "lop3.b32 v3, s3, %7, %8, 0xEA;\n\t"
      "mov.b32 {l0, h0}, v0;\n\tmov.b32 {l1, h1}, v1;\n\tmov.b32 {l2, h2}, v2;\n\tmov.b32 {l3, h3}, v3;\n\t"
      "mov.b32 {xl0, xh0}, %3;\n\tmov.b32 {xl1, xh1}, %4;\n\tmov.b32 {xl2, xh2}, %5;\n\tmov.b32 {xl3, xh3}, %6;\n\t"
      "fma.rn.f32.bf16 %0, xl0, l0, %0;\n\tfma.rn.f32.bf16 %1, xh0, h0, %1;\n\t"
      "fma.rn.f32.bf16 %0, xl1, l1, %0;\n\tfma.rn.f32.bf16 %1, xh1, h1, %1;\n\t"
      "fma.rn.f32.bf16 %0, xl2, l2, %0;\n\tfma.rn.f32.bf16 %1, xh2, h2, %1;\n\t"
      "fma.rn.f32.bf16 %0, xl3, l3, %0;\n\tfma.rn.f32.bf16 %1, xh3, h3, %1;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "r"(w), "r"(x0), "r"(x1), "r"(x2), "r"(x3), "r"(mask), "r"(magic));
}

// As word_dot_bf16, with all eight products into one accumulator.
__device__ __forceinline__ void word_dot_bf16_acc(uint32_t w, uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                                                  float& c, uint32_t mask, uint32_t magic) {
  asm("{\n\t.reg .b32 s1, s2, s3, v0, v1, v2, v3;\n\t"
      ".reg .b16 l0, h0, l1, h1, l2, h2, l3, h3, xl0, xh0, xl1, xh1, xl2, xh2, xl3, xh3;\n\t"
      "shr.b32 s1, %1, 4;\n\t"
      "shr.b32 s2, %1, 8;\n\t"
      "shr.b32 s3, %1, 12;\n\t"
      "lop3.b32 v0, %1, %6, %7, 0xEA;\n\t"
      "lop3.b32 v1, s1, %6, %7, 0xEA;\n\t"
      "lop3.b32 v2, s2, %6, %7, 0xEA;\n\t"
      "lop3.b32 v3, s3, %6, %7, 0xEA;\n\t"
      "mov.b32 {l0, h0}, v0;\n\tmov.b32 {l1, h1}, v1;\n\tmov.b32 {l2, h2}, v2;\n\tmov.b32 {l3, h3}, v3;\n\t"
      "mov.b32 {xl0, xh0}, %2;\n\tmov.b32 {xl1, xh1}, %3;\n\tmov.b32 {xl2, xh2}, %4;\n\tmov.b32 {xl3, xh3}, %5;\n\t"
      "fma.rn.f32.bf16 %0, xl0, l0, %0;\n\tfma.rn.f32.bf16 %0, xh0, h0, %0;\n\t"
      "fma.rn.f32.bf16 %0, xl1, l1, %0;\n\tfma.rn.f32.bf16 %0, xh1, h1, %0;\n\t"
      "fma.rn.f32.bf16 %0, xl2, l2, %0;\n\tfma.rn.f32.bf16 %0, xh2, h2, %0;\n\t"
      "fma.rn.f32.bf16 %0, xl3, l3, %0;\n\tfma.rn.f32.bf16 %0, xh3, h3, %0;\n\t}"
      : "+f"(c)
      : "r"(w), "r"(x0), "r"(x1), "r"(x2), "r"(x3), "r"(mask), "r"(magic));
}

// Packed fp32x2 fused multiply-add: (c0, c1) += (a0, a1) * (b0, b1).
__device__ __forceinline__ void ffma2(float& c0, float& c1, float a0, float a1, float b0, float b1) {
  asm("{ .reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%0, %1};\n\t"
      "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rc; }"
      : "+f"(c0), "+f"(c1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Packed fp32x2 add: (a0, a1) += (b0, b1).
__device__ __forceinline__ void fadd2(float& a0, float& a1, float b0, float b1) {
  asm("{ .reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\t"
      "mov.b64 {%0, %1}, ra; }"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}

// The eight codes of a packed word as exact fp32 values q0..q7, without
// shifting most of them: a nibble at bits p..p+3 is masked in place into the
// mantissa of 2^(23-p), where bit p weighs exactly 1, so the float equals
// 2^(23-p) + q; the offsets are then removed exactly, two at a time.  Bits
// 20..31 (q5..q7) are first shifted down by 12 to bits 8..19.
__device__ __forceinline__ void unpack_codes_f32(uint32_t w, float (&q)[8]) {
  const uint32_t ws = w >> 12;
  q[0] = __uint_as_float((w & 0x0000000Fu) | 0x4B000000u);   // 2^23 + q0
  q[1] = __uint_as_float((w & 0x000000F0u) | 0x49000000u);   // 2^19 + q1
  q[2] = __uint_as_float((w & 0x00000F00u) | 0x47000000u);   // 2^15 + q2
  q[3] = __uint_as_float((w & 0x0000F000u) | 0x45000000u);   // 2^11 + q3
  q[4] = __uint_as_float((w & 0x000F0000u) | 0x43000000u);   // 2^7  + q4
  q[5] = __uint_as_float((ws & 0x00000F00u) | 0x47000000u);  // 2^15 + q5
  q[6] = __uint_as_float((ws & 0x0000F000u) | 0x45000000u);  // 2^11 + q6
  q[7] = __uint_as_float((ws & 0x000F0000u) | 0x43000000u);  // 2^7  + q7
  fadd2(q[0], q[1], -8388608.f, -524288.f);
  fadd2(q[2], q[3], -32768.f, -2048.f);
  fadd2(q[4], q[5], -128.f, -32768.f);
  fadd2(q[6], q[7], -2048.f, -128.f);
}

// bf16x2 arithmetic (packed, one rounding per lane).
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

}  // namespace q4
