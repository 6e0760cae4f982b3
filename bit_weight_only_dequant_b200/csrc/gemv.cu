// Split-K weight-streaming GEMV for decode row counts (M <= 16) on sm_100a.
//
// Why this shape: at small M the matmul moves ~0.5 byte of packed weight per
// 2*M flops, so the time is the time to stream the weights from HBM once (the
// bandwidth argument of the blog post "One Config Line Made My 27B Model 2.7x
// Faster", section "Gotcha #2").  The kernel's job is to keep enough bytes in
// flight and to spend as few instructions per weight as possible turning
// nibbles into multiply operands: at 7+ TB/s a B200 SM has about two
// lane-instructions per weight.
//
// Structure (one CTA of 16 warps per SM):
//  * A CTA owns one K-slice and a contiguous range of 16-row bands.  Its
//    warps form a (Wn x Wk) grid: Wn bands in flight at a time, each band's
//    slice cut into Wk equal group-aligned pieces, one per warp, so every warp
//    streams the same number of bytes.  The Wk partial sums of a band are
//    added in piece order through shared memory (deterministic).
//  * The CTA copies its slice of the activations into shared memory, k
//    reordered inside every 16-block to match the packed operand fragments
//    (NVFP4: rows rescaled by a power of two into FP16).
//  * Each warp streams its pieces straight into registers: every lane loads
//    its 16 bytes of each 512-byte tile with a 128-bit read-only global load
//    (a warp load covers one whole tile), prefetched four 128-groups ahead, so
//    ~64 KB per SM are in flight without shared memory, TMA issue or barrier
//    polling on the weight stream.  The first loads are issued before the
//    activations are staged.
//  * Per 32-bit word (8 weights) a lane builds the A fragment of one
//    mma.sync m16n8k16 (16 output columns x 16 k): 3 shifts, 4 LOP3 and
//    4 exact BF16 subtractions (int4), or 4 hardware e2m1 -> f16 conversions
//    (NVFP4).  The activations are the n8 side: one MMA serves 8 rows.
//    Group scales multiply the fp32 MMA results (int4: once per 128-group,
//    NVFP4: once per 16-group).
//  * Split-K partials across CTAs go to a fp32 workspace; the last CTA to
//    finish a band (arrival counter) adds them in split order.
#include "common.cuh"
#include "kernels.h"

namespace w4 {

namespace {

#ifndef W4_GEMV_INT4_F16
#define W4_GEMV_INT4_F16 0
#endif
#ifndef W4_GEMV_PREFETCH
#define W4_GEMV_PREFETCH 4
#endif
// Activations go to the tensor cores as FP16 (rescaled per row slice) for
// NVFP4 always, and for int4 when W4_GEMV_INT4_F16 is set.
template <int FMT>
struct XF16 {
  static constexpr bool value = FMT == 1 || W4_GEMV_INT4_F16 != 0;
};
#ifndef W4_GEMV_WARPS
#define W4_GEMV_WARPS 16
#endif
constexpr int kWarps = W4_GEMV_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kPD = W4_GEMV_PREFETCH;                       // 128-groups in flight per warp
constexpr int kMaxMT = 2;                                    // M <= 16
constexpr int kRowWords = 64;                                // per-row words (M <= 64)
constexpr int kZeroOff = 2 * kRowWords * 4;                  // 128 zero bytes
constexpr int kRedOff = kZeroOff + 128;
constexpr int kRedBytes = kWarps * 32 * 4 * kMaxMT * 4;      // per-lane partial sums
constexpr int kHeaderBytes = kRedOff + kRedBytes;
constexpr int kMaxSmem = 232448;                             // 227 KB opt-in
static_assert(kHeaderBytes % 128 == 0, "activation image alignment");

struct Params {
  const __nv_bfloat16* x;
  const uint8_t* w;
  const uint8_t* s;
  const float* g;
  __nv_bfloat16* y;
  float* ws;
  unsigned* counters;
  unsigned* err;
  int M, N, K, NT, S, kslice, ctas_x, row_stride;  // row_stride in bytes
  int wn, wk;                                      // warp grid: bands x pieces
};

// Element kin of a 64-block sits at this element offset of the block's image
// in shared memory: lane t reads 16 contiguous elements k = 16 j + 4 t + e.
__device__ __forceinline__ int perm64(int kin) {
  const int j = kin >> 4, t = (kin >> 2) & 3, e = kin & 3;
  return t * 16 + j * 4 + e;
}

template <int FMT>
__device__ void stage_activations(const Params& p, int k_lo, int k_len, uint8_t* xs,
                                  float* row_mul, unsigned* row_aux) {
  const int tid = threadIdx.x;
  const int chunks_per_row = k_len / 8;  // 8 elements per 16-byte load
  if (XF16<FMT>::value) {
    if (tid < kRowWords) row_aux[tid] = 0u;
    __syncthreads();
    for (int m = 0; m < p.M; ++m) {
      float mx = 0.f;
      const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)m * p.K + k_lo);
      for (int c = tid; c < chunks_per_row; c += blockDim.x) {
        const uint4 v = src[c];
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mx = fmaxf(mx, fabsf(__uint_as_float(u[i] << 16)));
          mx = fmaxf(mx, fabsf(__uint_as_float(u[i] & 0xFFFF0000u)));
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if ((tid & 31) == 0) atomicMax(row_aux + m, __float_as_uint(mx));
    }
    __syncthreads();
    if (tid < p.M) {
      const float mx = __uint_as_float(row_aux[tid]);
      int e = 0;
      if (mx > 0.f && isfinite(mx)) e = ilogbf(mx) - 14;  // max * 2^-e in [2^14, 2^15)
      row_mul[tid] = ldexpf(1.f, e);
      row_aux[tid] = static_cast<unsigned>(-e);           // exponent applied to the row
    }
    __syncthreads();
  }
  for (int idx = tid; idx < p.M * chunks_per_row; idx += blockDim.x) {
    const int m = idx / chunks_per_row, c = idx - m * chunks_per_row;
    const uint4 v = reinterpret_cast<const uint4*>(p.x + (size_t)m * p.K + k_lo)[c];
    const int kin0 = c * 8;
    const int blk = kin0 >> 6, in = kin0 & 63;
    uint32_t out[4] = {v.x, v.y, v.z, v.w};
    if (XF16<FMT>::value) {
      const int sh = static_cast<int>(row_aux[m]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = ldexpf(__uint_as_float(out[i] << 16), sh);
        const float hi = ldexpf(__uint_as_float(out[i] & 0xFFFF0000u), sh);
        __half2 h = __floats2half2_rn(lo, hi);
        out[i] = *reinterpret_cast<uint32_t*>(&h);
      }
    }
    uint8_t* row = xs + (size_t)m * p.row_stride + blk * 128;
    *reinterpret_cast<uint2*>(row + perm64(in) * 2) = make_uint2(out[0], out[1]);
    *reinterpret_cast<uint2*>(row + perm64(in + 4) * 2) = make_uint2(out[2], out[3]);
  }
  __syncthreads();
}

// c = A . B (fresh accumulator), fp32
__device__ __forceinline__ void mma_bf16_first(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ void mma_f16_first(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Streaming read-only loads of the packed weights (read once: no L1 allocation,
// evict first from L2).
__device__ __forceinline__ uint4 ldg_stream16(const uint8_t* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint2 ldg_stream8(const uint8_t* p, uint64_t pol) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint32_t ldg_stream4(const uint8_t* p, uint64_t pol) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;"
               : "=r"(v)
               : "l"(p), "l"(pol));
  return v;
}

// One 128-group (two 64-blocks) of one band, int4.  w0/w1: this lane's words
// of the two tiles; sp: BF16 scales of rows g and g+8.
template <int MT>
__device__ __forceinline__ void group_int4(uint4 w0, uint4 w1, uint32_t sp,
                                           const uint8_t* const* xrow, const int* xstep, int kbl,
                                           float (*acc)[4]) {
  const float s_lo = __uint_as_float(sp << 16);          // row g
  const float s_hi = __uint_as_float(sp & 0xFFFF0000u);  // row g + 8
  float c[MT][4];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint4 wv = half ? w1 : w0;
    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t a[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (W4_GEMV_INT4_F16) {
        // FP16 holds two nibbles per 16-bit half in its mantissa: one shift per word
        const uint32_t hi = wd[j] >> 8;
        a[j][0] = int4_lo_pair_to_f16x2(wd[j]);
        a[j][1] = int4_hi_pair_to_f16x2(wd[j]);
        a[j][2] = int4_lo_pair_to_f16x2(hi);
        a[j][3] = int4_hi_pair_to_f16x2(hi);
      } else {
        a[j][0] = int4_pair_to_bf16x2(wd[j]);
        a[j][1] = int4_pair_to_bf16x2(wd[j] >> 4);
        a[j][2] = int4_pair_to_bf16x2(wd[j] >> 8);
        a[j][3] = int4_pair_to_bf16x2(wd[j] >> 12);
      }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const uint4* xb = reinterpret_cast<const uint4*>(xrow[mt] + (kbl + half) * xstep[mt]);
      const uint4 v0 = xb[0], v1 = xb[1];
      const uint32_t bx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (W4_GEMV_INT4_F16) {
          if (half == 0 && j == 0) mma_f16_first(c[mt], a[0], bx[0], bx[1]);
          else mma_f16_16816(c[mt], a[j], bx[2 * j], bx[2 * j + 1]);
        } else {
          if (half == 0 && j == 0) mma_bf16_first(c[mt], a[0], bx[0], bx[1]);
          else mma_bf16_16816(c[mt], a[j], bx[2 * j], bx[2 * j + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    acc[mt][0] = fmaf(s_lo, c[mt][0], acc[mt][0]);
    acc[mt][1] = fmaf(s_lo, c[mt][1], acc[mt][1]);
    acc[mt][2] = fmaf(s_hi, c[mt][2], acc[mt][2]);
    acc[mt][3] = fmaf(s_hi, c[mt][3], acc[mt][3]);
  }
}

// One 64-block of one band, NVFP4 (a scale per 16-group, i.e. per MMA).  wv:
// this lane's words of the tile; sv: E4M3 scales of rows g and g+8, 4 groups.
template <int MT>
__device__ __forceinline__ void block_nvfp4(uint4 wv, uint2 sv, const uint8_t* const* xrow,
                                            const int* xstep, int kbl, float (*acc)[4]) {
  const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
  uint32_t a[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    a[j][0] = e2m1x2_to_f16x2(wd[j]);
    a[j][1] = e2m1x2_to_f16x2(wd[j] >> 8);
    a[j][2] = e2m1x2_to_f16x2(wd[j] >> 16);
    a[j][3] = e2m1x2_to_f16x2(wd[j] >> 24);
  }
  const uint32_t sw2[2] = {sv.x, sv.y};
  float2 sf[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint16_t>(sw2[j >> 1] >> (16 * (j & 1))));
    sf[j] = __half22float2(*reinterpret_cast<const __half2*>(&s2));
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const uint4* xb = reinterpret_cast<const uint4*>(xrow[mt] + kbl * xstep[mt]);
    const uint4 v0 = xb[0], v1 = xb[1];
    const uint32_t bx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float c[4];
      mma_f16_first(c, a[j], bx[2 * j], bx[2 * j + 1]);
      acc[mt][0] = fmaf(sf[j].x, c[0], acc[mt][0]);
      acc[mt][1] = fmaf(sf[j].x, c[1], acc[mt][1]);
      acc[mt][2] = fmaf(sf[j].y, c[2], acc[mt][2]);
      acc[mt][3] = fmaf(sf[j].y, c[3], acc[mt][3]);
    }
  }
}

template <int FMT, int MT>
__device__ __forceinline__ void band_epilogue(const Params& p, int band, int split, int lane,
                                              const float* row_mul, const float (*vals)[4]) {
  const int g = lane >> 2, t = lane & 3;
  const float gmul = FMT == 1 ? __ldg(p.g) : 1.f;
  const int n0 = band * 16 + g;
  if (p.S == 1) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = mt * 8 + 2 * t + (i & 1);
        const int n = n0 + 8 * (i >> 1);
        if (m < p.M && n < p.N) {
          float v = vals[mt][i];
          if (XF16<FMT>::value) v = v * row_mul[m] * gmul;
          p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(v);
        }
      }
    return;
  }
  const size_t Npad = (size_t)p.NT * 16;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = mt * 8 + 2 * t + (i & 1);
      const int n = n0 + 8 * (i >> 1);
      if (m < p.M) {
        float v = vals[mt][i];
        if (XF16<FMT>::value) v = v * row_mul[m];
        __stcg(p.ws + ((size_t)split * p.M + m) * Npad + n, v);
      }
    }
  __threadfence();
  __syncwarp();
  unsigned prev = 0;
  if (lane == 0) prev = atomicAdd(p.counters + band, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != static_cast<unsigned>(p.S - 1)) return;
  __threadfence();
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = mt * 8 + 2 * t + (i & 1);
      const int n = n0 + 8 * (i >> 1);
      if (m < p.M && n < p.N) {
        float v = 0.f;
        for (int sp = 0; sp < p.S; ++sp) v += __ldcg(p.ws + ((size_t)sp * p.M + m) * Npad + n);
        p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(v * gmul);
      }
    }
  if (lane == 0) p.counters[band] = 0u;
}

// The words a lane needs for one 128-group of one band.
struct GroupWords {
  uint4 w0, w1;   // the two 64-blocks
  uint2 s0, s1;   // int4: s0.x = scales of rows g, g+8; NVFP4: per-block E4M3 scales
};

template <int FMT>
__device__ __forceinline__ GroupWords load_group(const Params& p, int band, int kb, int lane,
                                                 uint64_t pol) {
  GroupWords gw;
  const int g = lane >> 2;
  const uint8_t* wt = p.w + ((size_t)band * (p.K >> 6) + kb) * kTileBytes + lane * 16;
  gw.w0 = ldg_stream16(wt, pol);
  gw.w1 = ldg_stream16(wt + kTileBytes, pol);
  if (FMT == 0) {
    gw.s0.x = ldg_stream4(p.s + ((size_t)band * (p.K >> 7) + (kb >> 1)) * 32 + g * 4, pol);
    gw.s0.y = 0u;
    gw.s1 = make_uint2(0u, 0u);
  } else {
    const uint8_t* st = p.s + ((size_t)band * (p.K >> 6) + kb) * 64 + g * 8;
    gw.s0 = ldg_stream8(st, pol);
    gw.s1 = ldg_stream8(st + 64, pol);
  }
  return gw;
}

template <int FMT, int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* row_mul = reinterpret_cast<float*>(smem);
  unsigned* row_aux = reinterpret_cast<unsigned*>(smem + kRowWords * 4);
  const uint8_t* zero = smem + kZeroOff;
  float* red = reinterpret_cast<float*>(smem + kRedOff);
  uint8_t* xs = smem + kHeaderBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.y;
  const int k_lo = split * p.kslice;
  const int k_len = min(p.K - k_lo, p.kslice);
  const int band_lo = (int)(((long long)blockIdx.x * p.NT) / p.ctas_x);
  const int band_hi = (int)(((long long)(blockIdx.x + 1) * p.NT) / p.ctas_x);
  const int nbands = band_hi - band_lo;

  // warp grid: wi = band slot, wj = K piece of whole 128-groups
  const int wi = warp % p.wn, wj = warp / p.wn;
  const int groups = k_len >> 7;
  const int g_lo = wj * groups / p.wk, g_hi = (wj + 1) * groups / p.wk;
  const int ng = g_hi - g_lo;                  // 128-groups in this warp's piece
  const int kb_base = (k_lo >> 6) + 2 * g_lo;  // first 64-block (global) of the piece
  const int rounds = (nbands + p.wn - 1) / p.wn;
  const int my_rounds = wi < nbands ? (nbands - wi + p.wn - 1) / p.wn : 0;
  const uint64_t pol = policy_evict_first();

  // the first loads go out before the activations are staged
  GroupWords buf[kPD];
  if (my_rounds > 0) {
#pragma unroll
    for (int u = 0; u < kPD; ++u)
      if (u < ng) buf[u] = load_group<FMT>(p, band_lo + wi, kb_base + 2 * u, lane, pol);
  }

  if (threadIdx.x < 32) reinterpret_cast<uint32_t*>(smem + kZeroOff)[threadIdx.x] = 0u;
  stage_activations<FMT>(p, k_lo, k_len, xs, row_mul, row_aux);  // ends with __syncthreads

  // activation rows of this lane (row m = 8 mt + g); rows past M read zeros
  const uint8_t* xrow[MT];
  int xstep[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = mt * 8 + g;
    const bool real = m < p.M;
    xrow[mt] = real ? xs + (size_t)m * p.row_stride + t * 32 : zero;
    xstep[mt] = real ? 128 : 0;
  }
  const int kbl_base = 2 * g_lo;               // slice-local first 64-block of the piece

  for (int r = 0; r < rounds; ++r) {
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;
    const bool active = r < my_rounds;
    const int band = band_lo + wi + r * p.wn;
    if (active) {
      if (r > 0) {
#pragma unroll
        for (int u = 0; u < kPD; ++u)
          if (u < ng) buf[u] = load_group<FMT>(p, band, kb_base + 2 * u, lane, pol);
      }
      for (int gi0 = 0; gi0 < ng; gi0 += kPD) {
#pragma unroll
        for (int u = 0; u < kPD; ++u) {
          const int gi = gi0 + u;
          if (gi < ng) {
            const GroupWords cur = buf[u];
            if (gi + kPD < ng) buf[u] = load_group<FMT>(p, band, kb_base + 2 * (gi + kPD), lane, pol);
            const int kbl = kbl_base + 2 * gi;
            if (FMT == 0) {
              group_int4<MT>(cur.w0, cur.w1, cur.s0.x, xrow, xstep, kbl, acc);
            } else {
              block_nvfp4<MT>(cur.w0, cur.s0, xrow, xstep, kbl, acc);
              block_nvfp4<MT>(cur.w1, cur.s1, xrow, xstep, kbl + 1, acc);
            }
          }
        }
      }
    }
    if (p.wk == 1) {
      if (active) band_epilogue<FMT, MT>(p, band, split, lane, row_mul, acc);
      continue;
    }
    // add the wk pieces of each band in piece order
    float* mine = red + (warp * 32 + lane) * 4 * MT;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) mine[mt * 4 + i] = active ? acc[mt][i] : 0.f;
    __syncthreads();
    if (wj == 0 && active) {
      float sum[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sum[mt][i] = 0.f;
      for (int pc = 0; pc < p.wk; ++pc) {
        const float* o = red + ((pc * p.wn + wi) * 32 + lane) * 4 * MT;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) sum[mt][i] += o[mt * 4 + i];
      }
      band_epilogue<FMT, MT>(p, band, split, lane, row_mul, sum);
    }
    __syncthreads();
  }
}

template <int FMT, int MT>
cudaError_t launch_t(const GemvPlan& pl, const GemmArgs& a, cudaStream_t st) {
  Params p;
  p.x = static_cast<const __nv_bfloat16*>(a.x);
  p.w = static_cast<const uint8_t*>(a.w);
  p.s = static_cast<const uint8_t*>(a.s);
  p.g = a.g;
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.ws = a.ws;
  p.counters = a.counters;
  p.err = a.err;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.NT = (a.N + 15) / 16;
  p.S = pl.S;
  p.kslice = pl.kslice;
  p.ctas_x = pl.ctas_x;
  p.row_stride = (pl.kslice / 64) * 128 + 16;
  p.wn = pl.wn;
  p.wk = pl.wk;
  // raise the dynamic shared memory limit once per device (kept out of the
  // steady state so launches can be captured in CUDA graphs)
  static int smem_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem_set[dev] < pl.smem) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<FMT, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = kMaxSmem;
  }
  gemv_kernel<FMT, MT><<<dim3(pl.ctas_x, pl.S), kThreads, pl.smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Picks the K splits across CTAs (S) and the warp grid (wn bands x wk pieces)
// that minimise the largest number of 64-blocks any warp streams, with small
// penalties for cross-CTA split-K and per-round reductions.
GemvPlan plan_gemv(int fmt, int M, int N, int K, int num_sms) {
  (void)fmt;
  GemvPlan pl;
  pl.mt = M <= 8 ? 1 : 2;
  const int NT = (N + 15) / 16;
  const int groups = K / 128;
  const int xbudget = kMaxSmem - kHeaderBytes;
  const int max_groups = (xbudget / M - 16) / 256;
  const int s_min = (groups + max_groups - 1) / max_groups;
  double best = 1e300;
  pl.S = s_min;
  pl.wk = 1;
  for (int S = s_min; S <= groups && S <= 16; ++S) {
    const int gslice = (groups + S - 1) / S;
    if ((S - 1) * gslice >= groups) continue;  // an empty split
    int ctas = num_sms / S;
    if (ctas < 1) ctas = 1;
    if (ctas > NT) ctas = NT;
    const int bands_max = (NT + ctas - 1) / ctas;
    for (int wk = 1; wk <= kWarps; wk *= 2) {
      if (wk > gslice) break;
      if (kWarps % wk != 0) continue;
      const int wn = kWarps / wk;
      const int rounds = (bands_max + wn - 1) / wn;
      const int piece = 2 * ((gslice + wk - 1) / wk);
      double cost = (double)rounds * (piece + (wk > 1 ? 2.0 : 0.5)) + (S > 1 ? 3.0 : 0.0);
      if (cost < best - 1e-9) {
        best = cost;
        pl.S = S;
        pl.wk = wk;
      }
    }
  }
  pl.wn = kWarps / pl.wk;
  const int gslice = (groups + pl.S - 1) / pl.S;
  pl.kslice = gslice * 128;
  int ctas = num_sms / pl.S;
  if (ctas < 1) ctas = 1;
  if (ctas > NT) ctas = NT;
  pl.ctas_x = ctas;
  pl.smem = kHeaderBytes + M * ((pl.kslice / 64) * 128 + 16);
  return pl;
}

size_t gemv_workspace_floats(const GemvPlan& p, int M, int N) {
  return p.S > 1 ? static_cast<size_t>(p.S) * M * ((N + 15) / 16 * 16) : 0;
}

size_t gemv_counters(const GemvPlan& p, int N) { return p.S > 1 ? (N + 15) / 16 : 0; }

cudaError_t launch_gemv(const GemvPlan& p, const GemmArgs& a, cudaStream_t st) {
  if (a.fmt == 0) return p.mt == 1 ? launch_t<0, 1>(p, a, st) : launch_t<0, 2>(p, a, st);
  return p.mt == 1 ? launch_t<1, 1>(p, a, st) : launch_t<1, 2>(p, a, st);
}

}  // namespace w4
