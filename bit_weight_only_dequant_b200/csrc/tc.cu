// Tensor-core path for speculative-verify row counts (M = 9 .. 64) on sm_100a.
//
// At M = 64 the matmul does 256 flops per packed weight byte, close to the
// B200 ridge, so the multiply-adds belong on the 5th-generation tensor cores
// (the pages' remark that verifying several drafted tokens in one pass turns
// a bandwidth-bound step into a slightly compute-bound one: blog post "One
// Config Line Made My 27B Model 2.7x Faster", section "The fix").
//
// Structure (one persistent CTA per SM, 10 warps, 256-row x M tiles):
//  * warp 8 (producer): per 64-k block, one 2-D TMA load of the activation
//    tile (M rows, SWIZZLE_128B, rows past M zero-filled) and 1-D bulk copies
//    of the 16 packed 512-byte weight tiles and their scales into a 6-stage
//    shared-memory ring.
//  * warps 0-7 (dequant, then epilogue): each lane turns its 16 packed bytes
//    into 32 scaled operands in registers (int4: q -> BF16, times the BF16
//    group scale with one rounding, i.e. exactly W_deq; NVFP4: e2m1 -> FP16
//    times the E4M3 scale, exact) and writes them straight into tensor memory
//    with tcgen05.st 16x256b, whose register layout matches the packed pairs.
//    Shared memory never holds dequantised weights.
//  * warp 9 (MMA): tcgen05.mma kind::f16 with A (weights, 128 rows) read from
//    tensor memory and B (activations, K-major SW128) from shared memory,
//    accumulating fp32 D (128 lanes x Mpad columns) per 128-row half.
//  * epilogue: tcgen05.ld of D, BF16 stores (or fp32 split-K partials reduced
//    in split order by the last CTA of the tile).
// Tensor memory: D at columns [0, 128), six A stages of 2 x 32 columns at
// [128, 512).  Every mbarrier wait is bounded; a timeout raises the device
// error word, the CTA drains its copies and MMAs and frees tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace w4 {

namespace {

constexpr int kTcStages = 6;
constexpr int kDeqWarps = 8;
constexpr int kTcThreads = (kDeqWarps + 2) * 32;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTcTileRows = 256;  // 16 bands, two 128-row MMA tiles
constexpr int kWStage = 16 * kTileBytes;       // 8192
constexpr int kSStage = 16 * 64;               // scales (NVFP4 size; INT4 uses 32 per band)
constexpr int kTmemCols = 512;
constexpr int kAColBase = 128;
constexpr int kMinSmem = 120 * 1024;           // keeps one CTA (and one TMEM owner) per SM

struct TcParams {
  const uint8_t* w;
  const uint8_t* s;
  const float* g;
  const float* row_mul;    // NVFP4: per-row power-of-two activation scale
  __nv_bfloat16* y;
  float* ws;
  unsigned* counters;
  unsigned* err;
  int M, N, K, KB, NT, tiles, S, kbs, units;
};

// ------------------------------------------------------------------ tcgen05 wrappers

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] . B[smem desc]^T, kind::f16, one CTA.
__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
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

// Instruction descriptor: fp32 D, A/B type (0 f16, 1 bf16), both K-major, M=128, N=mpad.
__host__ __device__ constexpr uint32_t make_idesc(int ab_type, int mpad) {
  return (1u << 4) | ((uint32_t)ab_type << 7) | ((uint32_t)ab_type << 10) |
         ((uint32_t)(mpad >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
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
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, phase)) return true;
    if ((i & 255u) == 0u) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kSpinNanos) break;
    }
  }
  *abort_flag = 1;
  atomicOr(err, kErrTimeout);
  return false;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hmul2_f16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ------------------------------------------------------------------ the kernel

template <int FMT, int MPAD>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap xmap, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int kBStage = MPAD * 128;
  uint8_t* Bs = smem;
  uint8_t* Ws = Bs + kTcStages * kBStage;
  uint8_t* Ss = Ws + kTcStages * kWStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(Ss + kTcStages * kSStage);
  uint64_t* full = bars;
  uint64_t* afull = bars + kTcStages;
  uint64_t* freeb = bars + 2 * kTcStages;
  uint64_t* dfull = bars + 3 * kTcStages;
  uint64_t* dfree = dfull + 1;
  uint64_t* drain = dfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile unsigned* fix_word = reinterpret_cast<volatile unsigned*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(afull + i, kDeqWarps);
      mbar_init(freeb + i, kDeqWarps + 1);
    }
    mbar_init(dfull, 1);
    mbar_init(dfree, kDeqWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int last_use[kTcStages];
      for (int i = 0; i < kTcStages; ++i) last_use[i] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x) {
        const int tile = unit / p.S, split = unit - tile * p.S;
        const int kb_lo = split * p.kbs, kb_hi = min(p.KB, kb_lo + p.kbs);
        const int nb0 = tile * 16;
        const int nvalid = min(16, p.NT - nb0);
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
          const int s = it % kTcStages;
          const uint32_t u = it / kTcStages;
          if (u > 0 && !tc_wait(freeb + s, (u - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t sb = FMT == 0 ? 32u : 64u;
          mbar_arrive_expect_tx(full + s, kBStage + nvalid * (kTileBytes + sb));
          tma_load_2d(Bs + s * kBStage, &xmap, kb * 64, 0, full + s);
          for (int b = 0; b < nvalid; ++b) {
            const size_t nb = (size_t)(nb0 + b);
            bulk_g2s(Ws + s * kWStage + b * kTileBytes, p.w + (nb * p.KB + kb) * kTileBytes,
                     kTileBytes, full + s);
            const uint8_t* ssrc = FMT == 0 ? p.s + (nb * (p.K >> 7) + (kb >> 1)) * 32
                                           : p.s + (nb * p.KB + kb) * 64;
            bulk_g2s(Ss + s * kSStage + b * sb, ssrc, sb, full + s);
          }
          last_use[s] = (int)u;
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int s = 0; s < kTcStages; ++s)
        if (last_use[s] >= 0) mbar_wait(full + s, last_use[s] & 1, p.err);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(FMT == 0 ? 1 : 0, MPAD);
      uint32_t it = 0, unit_i = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++unit_i) {
        const int tile = unit / p.S, split = unit - tile * p.S;
        const int kb_lo = split * p.kbs, kb_hi = min(p.KB, kb_lo + p.kbs);
        (void)tile;
        if (unit_i > 0) {
          if (!tc_wait(dfree, (unit_i - 1) & 1, abort_flag, p.err)) break;
          tc_fence_after();
        }
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
          const int s = it % kTcStages;
          const uint32_t u = it / kTcStages;
          if (!tc_wait(afull + s, u & 1, abort_flag, p.err) ||
              !tc_wait(full + s, u & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bbase = smem_u32(Bs + s * kBStage);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t a = tmem + kAColBase + s * 64 + h * 32 + j * 8;
              umma_ts(tmem + h * 64, a, sw128_desc(bbase + j * 32), idesc,
                      (kb > kb_lo || j > 0) ? 1u : 0u);
            }
          }
          umma_commit(freeb + s);
        }
        if (ok) umma_commit(dfull);
      }
      // drain: all issued MMAs complete before tensor memory is released
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- dequant + epilogue
    const int h = warp >> 2, q = warp & 3;
    const int g = lane >> 2;
    uint32_t it = 0, unit_i = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++unit_i) {
      const int tile = unit / p.S, split = unit - tile * p.S;
      const int kb_lo = split * p.kbs, kb_hi = min(p.KB, kb_lo + p.kbs);
      for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
        const int s = it % kTcStages;
        const uint32_t u = it / kTcStages;
        if (!tc_wait(full + s, u & 1, abort_flag, p.err) ||
            (u > 0 && !tc_wait(freeb + s, (u - 1) & 1, abort_flag, p.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[2][16];
#pragma unroll
        for (int bp = 0; bp < 2; ++bp) {
          const int band = h * 8 + 2 * q + bp;
          const uint4 wv =
              *reinterpret_cast<const uint4*>(Ws + s * kWStage + band * kTileBytes + lane * 16);
          const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
          if (FMT == 0) {
            const uint32_t sp = *reinterpret_cast<const uint32_t*>(Ss + s * kSStage + band * 32 + g * 4);
            const uint32_t s_lo = prmt(sp, sp, 0x1010u);  // (s_g, s_g)
            const uint32_t s_hi = prmt(sp, sp, 0x3232u);  // (s_g8, s_g8)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // register order of 16x256b: (row g, col 2t), (row g, col 2t+1),
              // (row g+8, col 2t), (row g+8, col 2t+1) = P0, P2, P1, P3
              r[bp][4 * j + 0] = hmul2_bf16(int4_pair_to_bf16x2(wd[j]), s_lo);
              r[bp][4 * j + 1] = hmul2_bf16(int4_pair_to_bf16x2(wd[j] >> 8), s_lo);
              r[bp][4 * j + 2] = hmul2_bf16(int4_pair_to_bf16x2(wd[j] >> 4), s_hi);
              r[bp][4 * j + 3] = hmul2_bf16(int4_pair_to_bf16x2(wd[j] >> 12), s_hi);
            }
          } else {
            const uint2 sv = *reinterpret_cast<const uint2*>(Ss + s * kSStage + band * 64 + g * 8);
            const uint32_t sw2[2] = {sv.x, sv.y};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t s2 =
                  e4m3x2_to_f16x2(static_cast<uint16_t>(sw2[j >> 1] >> (16 * (j & 1))));
              const uint32_t s_lo = prmt(s2, s2, 0x1010u), s_hi = prmt(s2, s2, 0x3232u);
              r[bp][4 * j + 0] = hmul2_f16(e2m1x2_to_f16x2(wd[j]), s_lo);
              r[bp][4 * j + 1] = hmul2_f16(e2m1x2_to_f16x2(wd[j] >> 16), s_lo);
              r[bp][4 * j + 2] = hmul2_f16(e2m1x2_to_f16x2(wd[j] >> 8), s_hi);
              r[bp][4 * j + 3] = hmul2_f16(e2m1x2_to_f16x2(wd[j] >> 24), s_hi);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(freeb + s);  // this warp's shared-memory reads are done
#pragma unroll
        for (int bp = 0; bp < 2; ++bp) {
          const uint32_t taddr = tmem + ((uint32_t)(32 * q + 16 * bp) << 16) + kAColBase + s * 64 + h * 32;
          tmem_st_16x256b_x4(taddr, r[bp]);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull + s);
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue of a unit
      if (!tc_wait(dfull, unit_i & 1, abort_flag, p.err)) break;
      tc_fence_after();
      float v[MPAD];
#pragma unroll
      for (int c = 0; c < MPAD / 16; ++c)
        tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + h * 64 + c * 16, v + 16 * c);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dfree);

      const int n = tile * kTcTileRows + h * 128 + 32 * q + lane;
      float gmul = 1.f;
      if (FMT == 1) gmul = __ldg(p.g);
      if (p.S == 1) {
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < MPAD; ++m) {
            if (m < p.M) {
              float val = v[m];
              if (FMT == 1) val = val * __ldg(p.row_mul + m) * gmul;
              p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(val);
            }
          }
        }
      } else {
        const size_t Npad = (size_t)p.NT * 16;
        if (n < p.N) {
#pragma unroll
          for (int m = 0; m < MPAD; ++m)
            if (m < p.M) __stcg(p.ws + ((size_t)split * p.M + m) * Npad + n, v[m]);
        }
        __threadfence();
        asm volatile("bar.sync 1, %0;" ::"n"(kDeqWarps * 32));
        if (threadIdx.x == 0) *fix_word = atomicAdd(p.counters + tile, 1u);
        asm volatile("bar.sync 1, %0;" ::"n"(kDeqWarps * 32));
        if (*fix_word == static_cast<unsigned>(p.S - 1)) {
          __threadfence();
          if (n < p.N) {
            for (int m = 0; m < p.M; ++m) {
              float acc = 0.f;
              for (int sp = 0; sp < p.S; ++sp) acc += __ldcg(p.ws + ((size_t)sp * p.M + m) * Npad + n);
              if (FMT == 1) acc = acc * __ldg(p.row_mul + m) * gmul;
              p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(acc);
            }
          }
          if (threadIdx.x == 0) p.counters[tile] = 0u;
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// Per-row power-of-two rescaling of the activations into FP16 (NVFP4 path):
// row_mul[m] = 2^e with max|x[m]| * 2^-e in [2^14, 2^15).
__global__ void prep_x_f16_kernel(const __nv_bfloat16* __restrict__ x, __half* __restrict__ xh,
                                  float* __restrict__ row_mul, int K) {
  const int m = blockIdx.x;
  const __nv_bfloat16* row = x + (size_t)m * K;
  float mx = 0.f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) mx = fmaxf(mx, fabsf(__bfloat162float(row[k])));
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    mx = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (threadIdx.x == 0) red[0] = mx;
  }
  __syncthreads();
  mx = red[0];
  int e = 0;
  if (mx > 0.f && isfinite(mx)) e = ilogbf(mx) - 14;
  if (threadIdx.x == 0) row_mul[m] = ldexpf(1.f, e);
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    xh[(size_t)m * K + k] = __float2half_rn(ldexpf(__bfloat162float(row[k]), -e));
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_xmap(CUtensorMap* map, const void* x, int M, int K, int mpad, bool f16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)mpad};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int FMT, int MPAD>
cudaError_t launch_t(const TcPlan& pl, const GemmArgs& a, const void* xsrc, const float* row_mul,
                     cudaStream_t st) {
  CUtensorMap map;
  if (!make_xmap(&map, xsrc, a.M, a.K, MPAD, FMT == 1)) return cudaErrorInvalidValue;
  TcParams p;
  p.w = static_cast<const uint8_t*>(a.w);
  p.s = static_cast<const uint8_t*>(a.s);
  p.g = a.g;
  p.row_mul = row_mul;
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.ws = a.ws;
  p.counters = a.counters;
  p.err = a.err;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.KB = a.K / 64;
  p.NT = (a.N + 15) / 16;
  p.tiles = (a.N + kTcTileRows - 1) / kTcTileRows;
  p.S = pl.S;
  p.kbs = pl.kbs;
  p.units = p.tiles * pl.S;
  static int smem_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem_set[dev] < pl.smem) {
    cudaError_t e =
        cudaFuncSetAttribute(tc_kernel<FMT, MPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = pl.smem;
  }
  tc_kernel<FMT, MPAD><<<pl.grid, kTcThreads, pl.smem, st>>>(map, p);
  return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const TcPlan& pl, const GemmArgs& a, const void* xsrc, const float* rm,
                       cudaStream_t st) {
  switch (pl.mpad) {
    case 16: return launch_t<FMT, 16>(pl, a, xsrc, rm, st);
    case 32: return launch_t<FMT, 32>(pl, a, xsrc, rm, st);
    case 48: return launch_t<FMT, 48>(pl, a, xsrc, rm, st);
    default: return launch_t<FMT, 64>(pl, a, xsrc, rm, st);
  }
}

}  // namespace

TcPlan plan_tc(int fmt, int M, int N, int K, int num_sms) {
  TcPlan pl;
  pl.mpad = (M + 15) / 16 * 16;
  const int tiles = (N + kTcTileRows - 1) / kTcTileRows;
  const int KB = K / 64;
  double best = 1e300;
  int best_s = 1;
  for (int S = 1; S <= 16 && S <= KB; ++S) {
    const int kbs = (KB + S - 1) / S;
    if ((S - 1) * kbs >= KB) continue;
    const int units = tiles * S;
    const int waves = (units + num_sms - 1) / num_sms;
    const double cost = (double)waves * kbs + (S > 1 ? 2.0 : 0.0);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = S;
    }
  }
  pl.S = best_s;
  pl.kbs = (KB + pl.S - 1) / pl.S;
  pl.units = tiles * pl.S;
  pl.grid = pl.units < num_sms ? pl.units : num_sms;
  int smem = kTcStages * (pl.mpad * 128 + kWStage + kSStage) + 256 + 1024;
  if (smem < kMinSmem) smem = kMinSmem;
  pl.smem = smem;
  (void)fmt;
  return pl;
}

size_t tc_workspace_floats(const TcPlan& p, int M, int N) {
  return p.S > 1 ? static_cast<size_t>(p.S) * M * ((N + 15) / 16 * 16) : 0;
}

size_t tc_counters(const TcPlan& p, int N) { return p.S > 1 ? (N + 15) / 16 : 0; }

size_t tc_x_f16_bytes(int fmt, int M, int K) {
  return fmt == 1 ? (size_t)M * K * 2 + 64 * sizeof(float) : 0;
}

cudaError_t launch_tc(const TcPlan& pl, const GemmArgs& a, void* xf16_scratch, cudaStream_t st) {
  if (a.fmt == 0) return launch_fmt<0>(pl, a, a.x, nullptr, st);
  __half* xh = static_cast<__half*>(xf16_scratch);
  float* rm = reinterpret_cast<float*>(static_cast<uint8_t*>(xf16_scratch) + (size_t)a.M * a.K * 2);
  prep_x_f16_kernel<<<a.M, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a.x), xh, rm, a.K);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_fmt<1>(pl, a, xh, rm, st);
}

}  // namespace w4
