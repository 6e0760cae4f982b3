// Device helpers shared by the kernels: status word, bounded mbarrier waits,
// the L2 eviction policy, bit-level unpacking and warp-level MMA wrappers (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.h"

namespace w4 {

// Error word set by kernels that give up a bounded wait.  Read and cleared by
// w4a16_device_status().
constexpr unsigned kErrTimeout = 1u;

// Bounds of every spin on an mbarrier: 2^31 polls or about two seconds of
// SM clock (checked every 1024 polls with clock64, which is cheap), far
// above the longest legitimate wait (microseconds).
constexpr uint32_t kSpinLimit = 1u << 31;
constexpr long long kSpinCycles = 4000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and records the timeout) if the phase does not
// complete within the bounds above.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, unsigned* err) {
  if (mbar_try_wait(bar, phase)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, phase)) return true;
    if ((i & 1023u) == 0u && clock64() - t0 > kSpinCycles) break;
  }
  atomicOr(err, kErrTimeout);
  return false;
}

// ------------------------------------------------------------------ L2 policy

// The streamed weights are read exactly once: evict them from L2 first.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------------ bit tricks

// (a & MASK) | MAGIC with both constants as instruction immediates
template <uint32_t MASK, uint32_t MAGIC>
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "n"(MAGIC));
  return d;
}

// Two int4 codes u (nibbles at bits 0..3 and 16..19 of `w`) -> BF16 pair of
// q = u - 8, exact.  0x4300 is BF16 128.0 whose last mantissa bit weighs 1, so
// OR-ing a nibble into it gives 128 + u; subtracting 136 leaves q.
__device__ __forceinline__ uint32_t int4_pair_to_bf16x2(uint32_t w) {
  const uint32_t v = lop3_and_or<0x000F000Fu, 0x43004300u>(w);
  uint32_t d;
  const uint32_t bias = 0x43084308u;  // BF16 136.0, twice
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(bias));
  return d;
}

// FP16 forms of the same conversion.  0x6400 is FP16 1024.0 with a mantissa
// LSB of 1 and ten mantissa bits, so a nibble at bits 0..3 gives 1024 + u and
// a nibble at bits 4..7 gives 1024 + 16 u; exact arithmetic then leaves q.
__device__ __forceinline__ uint32_t int4_lo_pair_to_f16x2(uint32_t w) {
  const uint32_t v = lop3_and_or<0x000F000Fu, 0x64006400u>(w);
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(v), "r"(0x64086408u));  // - 1032
  return d;
}
__device__ __forceinline__ uint32_t int4_hi_pair_to_f16x2(uint32_t w) {
  const uint32_t v = lop3_and_or<0x00F000F0u, 0x64006400u>(w);
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(v), "r"(0x2C002C00u), "r"(0xD480D480u));  // /16 - 72
  return d;
}

// Byte of two e2m1 codes (low nibble first, in the low 8 bits) -> f16x2, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low_bits) {
  uint32_t d;
  const uint16_t h = static_cast<uint16_t>(byte_in_low_bits & 0xFFu);
  asm("{\n\t.reg .b8 lo, hi;\n\t"
      "mov.b16 {lo, hi}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, lo;\n\t}"
      : "=r"(d)
      : "h"(h));
  return d;
}

// Two E4M3 bytes (low byte first) -> f16x2, exact (every finite E4M3 value is an FP16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t two) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(two));
  return d;
}

// ------------------------------------------------------------------ warp MMA (m16n8k16, fp32 acc)

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float* c, const uint32_t* a, uint32_t b0,
                                              uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ misc

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // RNE
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace w4


// SiLU(z) = z * sigmoid(z) = z / (1 + e^-z) in fp32 for the fused gate/up
// epilogues: the hardware exponential and a correctly rounded reciprocal
// (relative error a few 1e-6, far inside the layer's tolerance).  e^-z
// overflows to +inf for z below about -88, and z * (1 / inf) is -0, the limit.
__device__ __forceinline__ float silu_f32(float z) { return z * __frcp_rn(1.f + __expf(-z)); }
