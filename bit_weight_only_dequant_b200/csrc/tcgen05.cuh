// tcgen05, TMA and mbarrier-wait helpers shared by the tensor-core kernels
// (tc.cu: W4A16 with A in tensor memory; bs.cu: W4A4 block-scaled).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace w4 {

namespace {

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}


__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

template <int NC>
__device__ __forceinline__ void tmem_ld_32x32b(uint32_t taddr, float* v);

template <>
__device__ __forceinline__ void tmem_ld_32x32b<4>(uint32_t taddr, float* v) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

template <>
__device__ __forceinline__ void tmem_ld_32x32b<8>(uint32_t taddr, float* v) {
  tmem_ld_32x32b_x8(taddr, v);
}

template <>
__device__ __forceinline__ void tmem_ld_32x32b<16>(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <>
__device__ __forceinline__ void tmem_ld_32x32b<32>(uint32_t taddr, float* v) {
  tmem_ld_32x32b<16>(taddr, v);
  tmem_ld_32x32b<16>(taddr + 16, v + 16);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// K-major operand tile with 128-byte swizzle: rows of 64 16-bit elements,
// 8-row atoms 1024 bytes apart (SBO), leading offset unused (1), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                // LBO (16 bytes, ignored for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;      // SBO
  d |= (uint64_t)1u << 46;                // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                // SWIZZLE_128B
  return d;
}


__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait that also gives up when another role has already aborted.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t phase, volatile int* abort_flag,
                                        unsigned* err) {
  if (mbar_try_wait(bar, phase)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, phase)) return true;
    if ((i & 1023u) == 0u) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kSpinCycles) break;
    }
  }
  *abort_flag = 1;
  atomicOr(err, kErrTimeout);
  return false;
}


__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Warp-wide bounded wait: the warp proceeds together once the phase completes.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t phase, volatile int* abort_flag,
                                          unsigned* err) {
  // every lane polls the barrier itself: cheaper than one lane polling and a
  // shuffle broadcasting the result (measured: 7-17 % faster kernels)
  const bool ok = tc_wait(bar, phase, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

}  // namespace

// The driver's tensor-map encoder, looked up once (thread-safe static initialisation).
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

}  // namespace w4
