// Split-K weight-streaming GEMV for decode row counts on sm_100a.
//
// Why this shape: at M <= 16 the matmul moves ~0.5 byte of packed weight per
// 2*M flops, so the time is the time to stream the weights from HBM once (the
// bandwidth argument of the blog post "One Config Line Made My 27B Model 2.7x
// Faster", section "Gotcha #2").  The kernel's job is to keep enough bytes in
// flight and to spend as few instructions per weight as possible on turning
// nibbles into multiply operands: B200 issues ~2 lane-instructions per weight
// at full HBM speed.
//
// Structure (one CTA per SM, 8 worker warps, no producer warp):
//  * Each CTA owns one K-slice [k_lo, k_hi) and a contiguous range of 16-row
//    bands.  It first copies its slice of the activations into shared memory
//    (k reordered inside every 16-block to match the operand fragments of the
//    packed layout); NVFP4 rows are rescaled by a power of two into FP16.
//  * Each warp streams its bands' packed weights and scales through a private
//    3-stage ring of 4.5 KB stages filled by 1-D bulk copies (TMA) completing
//    on mbarriers, so ~64-96 KB per SM are in flight.
//  * Per 32-bit word (8 weights) a lane builds the A fragment of one
//    mma.sync m16n8k16 (rows = 16 output columns, k = 16) with 3 shifts,
//    4 LOP3 and 4 BF16 subtractions (int4), or 4 hardware e2m1 -> f16
//    conversions (NVFP4); the activations are the n8 side, so every MMA
//    serves M <= 8 rows at once.  Group scales are applied to the fp32 MMA
//    results (per 128-group for int4, per 16-group for NVFP4).
//  * Split-K partials go to a fp32 workspace; the last warp to finish a band
//    (arrival counter) adds the S partials in split order and writes BF16, so
//    the result does not depend on arrival order.
#include "common.cuh"
#include "kernels.h"

namespace w4 {

namespace {

#ifndef W4_GEMV_WARPS
#define W4_GEMV_WARPS 8
#endif
#ifndef W4_GEMV_STAGES
#define W4_GEMV_STAGES 3
#endif
#ifndef W4_GEMV_STAGE_KB
#define W4_GEMV_STAGE_KB 8
#endif
constexpr int kWarps = W4_GEMV_WARPS;
constexpr int kStages = W4_GEMV_STAGES;
constexpr int kStageKB = W4_GEMV_STAGE_KB;                   // k64 blocks per stage
constexpr int kStageWBytes = kStageKB * kTileBytes;         // 4096
constexpr int kStageSBytes = kStageKB * 64;                  // scales, room for NVFP4
constexpr int kStageBytes = kStageWBytes + kStageSBytes;    // 4608
constexpr int kBarBytes = (kWarps * kStages * 8 + 127) / 128 * 128;
constexpr int kHeaderBytes = kBarBytes + 512;                // mbarriers + 2 x 64 row words
constexpr int kMaxSmem = 232448;                             // 227 KB opt-in

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
};

// Element k of a 64-block (local index kin) sits at this element offset of
// the block's 64-element image in shared memory: lane t = (kin % 16) / 4
// reads elements [16 t, 16 t + 16) as k = 16 j + 4 t + e, e = 0..3, j = 0..3.
__device__ __forceinline__ int perm64(int kin) {
  const int j = kin >> 4, t = (kin >> 2) & 3, e = kin & 3;
  return t * 16 + j * 4 + e;
}

template <int FMT>
__device__ void stage_activations(const Params& p, int k_lo, int k_len, uint8_t* xs,
                                  float* row_mul, unsigned* row_max_bits) {
  const int tid = threadIdx.x;
  const int chunks_per_row = k_len / 8;  // 8 elements per 16-byte load
  if (FMT == 1) {
    // per-row largest magnitude over the slice
    if (tid < 64) row_max_bits[tid] = 0u;
    __syncthreads();
    for (int m = 0; m < p.M; ++m) {
      float mx = 0.f;
      const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)m * p.K + k_lo);
      for (int c = tid; c < chunks_per_row; c += blockDim.x) {
        uint4 v = src[c];
        const uint32_t* u = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mx = fmaxf(mx, fabsf(__uint_as_float(u[i] << 16)));
          mx = fmaxf(mx, fabsf(__uint_as_float(u[i] & 0xFFFF0000u)));
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if ((tid & 31) == 0) atomicMax(row_max_bits + m, __float_as_uint(mx));
    }
    __syncthreads();
    if (tid < p.M) {
      const float mx = __uint_as_float(row_max_bits[tid]);
      int e = 0;
      if (mx > 0.f && isfinite(mx)) e = ilogbf(mx) - 14;  // max * 2^-e in [2^14, 2^15)
      row_mul[tid] = ldexpf(1.f, e);
      row_max_bits[tid] = static_cast<unsigned>(-e);       // reused: exponent to apply
    }
    __syncthreads();
  }
  for (int idx = tid; idx < p.M * chunks_per_row; idx += blockDim.x) {
    const int m = idx / chunks_per_row, c = idx - m * chunks_per_row;
    const uint4 v = reinterpret_cast<const uint4*>(p.x + (size_t)m * p.K + k_lo)[c];
    const int kin0 = c * 8;              // slice-local k of the first element
    const int blk = kin0 >> 6, in = kin0 & 63;
    uint32_t out[4];
    const uint32_t* u = reinterpret_cast<const uint32_t*>(&v);
    if (FMT == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = u[i];
    } else {
      const int sh = static_cast<int>(row_max_bits[m]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = ldexpf(__uint_as_float(u[i] << 16), sh);
        const float hi = ldexpf(__uint_as_float(u[i] & 0xFFFF0000u), sh);
        __half2 h = __floats2half2_rn(lo, hi);
        out[i] = *reinterpret_cast<uint32_t*>(&h);
      }
    }
    // elements in..in+3 and in+4..in+7 each land on 4 contiguous slots
    uint8_t* row = xs + (size_t)m * p.row_stride + blk * 128;
    *reinterpret_cast<uint2*>(row + perm64(in) * 2) = make_uint2(out[0], out[1]);
    *reinterpret_cast<uint2*>(row + perm64(in + 4) * 2) = make_uint2(out[2], out[3]);
  }
  __syncthreads();
}

template <int FMT, int MT>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);                 // kWarps * kStages
  float* row_mul = reinterpret_cast<float*>(smem + kBarBytes);        // W4A16_MAX_M
  unsigned* row_aux = reinterpret_cast<unsigned*>(smem + kBarBytes + 256);
  uint8_t* ring = smem + kHeaderBytes;
  uint8_t* xs = ring + kWarps * kStages * kStageBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.y;
  const int k_lo = split * p.kslice;
  const int k_len = min(p.K - k_lo, p.kslice);
  const int nkb = k_len >> 6;                                          // 64-blocks in the slice
  const int band_lo = (int)(((long long)blockIdx.x * p.NT) / p.ctas_x);
  const int band_hi = (int)(((long long)(blockIdx.x + 1) * p.NT) / p.ctas_x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWarps * kStages; ++i) mbar_init(bars + i, 1);
    fence_mbar_init();
  }
  stage_activations<FMT>(p, k_lo, k_len, xs, row_mul, row_aux);  // ends with __syncthreads

  // This warp's bands: band_lo + warp, + kWarps, ...
  const int my_first = band_lo + warp;
  const int my_bands = my_first < band_hi ? (band_hi - my_first + kWarps - 1) / kWarps : 0;
  const int stages_per_band = (nkb + kStageKB - 1) / kStageKB;
  const int total = my_bands * stages_per_band;
  uint64_t* my_bars = bars + warp * kStages;
  uint8_t* my_ring = ring + warp * kStages * kStageBytes;
  const int KB = p.K >> 6;
  const uint64_t pol = policy_evict_first();

  auto issue = [&](int L) {
    const int bi = L / stages_per_band, st = L - bi * stages_per_band;
    const int band = my_first + bi * kWarps;
    const int kb0 = (k_lo >> 6) + st * kStageKB;
    const int nblk = min(kStageKB, nkb - st * kStageKB);
    const int buf = L % kStages;
    uint8_t* dst = my_ring + buf * kStageBytes;
    const uint8_t* wsrc = p.w + ((size_t)band * KB + kb0) * kTileBytes;
    uint32_t sbytes;
    const uint8_t* ssrc;
    if (FMT == 0) {
      sbytes = nblk * 16;  // 32 bytes per 128-group = 2 blocks
      ssrc = p.s + ((size_t)band * (p.K >> 7) + (kb0 >> 1)) * 32;
    } else {
      sbytes = nblk * 64;
      ssrc = p.s + ((size_t)band * KB + kb0) * 64;
    }
    mbar_arrive_expect_tx(my_bars + buf, nblk * kTileBytes + sbytes);
    bulk_g2s_evict_first(dst, wsrc, nblk * kTileBytes, my_bars + buf, pol);
    bulk_g2s_evict_first(dst + kStageWBytes, ssrc, sbytes, my_bars + buf, pol);
  };

  if (lane == 0) {
    for (int L = 0; L < min(kStages, total); ++L) issue(L);
  }

  float acc[MT][4];
  float cg[MT][2][4];
  bool failed = false;
  int L = 0;
  for (int bi = 0; bi < my_bands && !failed; ++bi) {
    const int band = my_first + bi * kWarps;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;

    for (int st = 0; st < stages_per_band; ++st, ++L) {
      const int buf = L % kStages;
      if (!mbar_wait(my_bars + buf, (L / kStages) & 1, p.err)) {
        failed = true;
        break;
      }
      const uint8_t* sw = my_ring + buf * kStageBytes;
      const uint8_t* ss = sw + kStageWBytes;
      const int nblk = min(kStageKB, nkb - st * kStageKB);
      for (int bb = 0; bb < nblk; ++bb) {
        const int kbl = st * kStageKB + bb;  // slice-local 64-block
        const uint4 wv = *reinterpret_cast<const uint4*>(sw + bb * kTileBytes + lane * 16);
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
        // A fragments of the four k16 sub-blocks (pairs P0..P3 = a0..a3)
        uint32_t a[4][4];
        if (FMT == 0) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a[j][0] = int4_pair_to_bf16x2(wd[j]);
            a[j][1] = int4_pair_to_bf16x2(wd[j] >> 4);
            a[j][2] = int4_pair_to_bf16x2(wd[j] >> 8);
            a[j][3] = int4_pair_to_bf16x2(wd[j] >> 12);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a[j][0] = e2m1x2_to_f16x2(wd[j]);
            a[j][1] = e2m1x2_to_f16x2(wd[j] >> 8);
            a[j][2] = e2m1x2_to_f16x2(wd[j] >> 16);
            a[j][3] = e2m1x2_to_f16x2(wd[j] >> 24);
          }
        }
        const int half = kbl & 1;  // int4: which 64-block of the 128-group
        float2 sf[4];              // nvfp4: (row g, row g+8) scale of each k16 group
        if (FMT == 1) {
          const uint2 sv = *reinterpret_cast<const uint2*>(ss + bb * 64 + g * 8);
          const uint32_t sw2[2] = {sv.x, sv.y};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t s2 =
                e4m3x2_to_f16x2(static_cast<uint16_t>(sw2[j >> 1] >> (16 * (j & 1))));
            sf[j] = __half22float2(*reinterpret_cast<const __half2*>(&s2));
          }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          // activation fragments of row m = 8 mt + g: words (j, pair)
          uint32_t bx[8];
          const int m = mt * 8 + g;
          if (m < p.M) {
            const uint4* src =
                reinterpret_cast<const uint4*>(xs + (size_t)m * p.row_stride + kbl * 128 + t * 32);
            const uint4 v0 = src[0], v1 = src[1];
            bx[0] = v0.x; bx[1] = v0.y; bx[2] = v0.z; bx[3] = v0.w;
            bx[4] = v1.x; bx[5] = v1.y; bx[6] = v1.z; bx[7] = v1.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) bx[i] = 0u;
          }
          if (FMT == 0) {
            if (half == 0) {
#pragma unroll
              for (int i = 0; i < 4; ++i) cg[mt][0][i] = cg[mt][1][i] = 0.f;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) mma_bf16_16816(cg[mt][half], a[j], bx[2 * j], bx[2 * j + 1]);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float c[4] = {0.f, 0.f, 0.f, 0.f};
              mma_f16_16816(c, a[j], bx[2 * j], bx[2 * j + 1]);
              acc[mt][0] = fmaf(sf[j].x, c[0], acc[mt][0]);
              acc[mt][1] = fmaf(sf[j].x, c[1], acc[mt][1]);
              acc[mt][2] = fmaf(sf[j].y, c[2], acc[mt][2]);
              acc[mt][3] = fmaf(sf[j].y, c[3], acc[mt][3]);
            }
          }
        }
        if (FMT == 0 && half == 1) {
          // fold the group: acc += s_row * (sum over the 128 k of q x)
          const uint32_t sp = *reinterpret_cast<const uint32_t*>(ss + (bb >> 1) * 32 + g * 4);
          const float s_lo = __uint_as_float(sp << 16);           // row g
          const float s_hi = __uint_as_float(sp & 0xFFFF0000u);   // row g + 8
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            acc[mt][0] = fmaf(s_lo, cg[mt][0][0] + cg[mt][1][0], acc[mt][0]);
            acc[mt][1] = fmaf(s_lo, cg[mt][0][1] + cg[mt][1][1], acc[mt][1]);
            acc[mt][2] = fmaf(s_hi, cg[mt][0][2] + cg[mt][1][2], acc[mt][2]);
            acc[mt][3] = fmaf(s_hi, cg[mt][0][3] + cg[mt][1][3], acc[mt][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0 && L + kStages < total) issue(L + kStages);
    }
    if (failed) break;

    // ---------------------------------------------------------------- epilogue of a band
    // lane holds rows n = 16 band + g (+8) and activation rows m = 8 mt + 2t (+1)
    float gmul = 1.f;
    if (FMT == 1) gmul = __ldg(p.g);
    const int n0 = band * 16 + g;
    if (p.S == 1) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = mt * 8 + 2 * t + (i & 1);
          const int n = n0 + 8 * (i >> 1);
          if (m < p.M && n < p.N) {
            float v = acc[mt][i];
            if (FMT == 1) v = v * row_mul[m] * gmul;
            p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(v);
          }
        }
      }
    } else {
      const int Npad = p.NT * 16;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = mt * 8 + 2 * t + (i & 1);
          const int n = n0 + 8 * (i >> 1);
          if (m < p.M) {
            float v = acc[mt][i];
            if (FMT == 1) v = v * row_mul[m];
            __stcg(p.ws + ((size_t)split * p.M + m) * Npad + n, v);
          }
        }
      }
      __threadfence();
      __syncwarp();
      unsigned prev = 0;
      if (lane == 0) prev = atomicAdd(p.counters + band, 1u);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev == static_cast<unsigned>(p.S - 1)) {
        __threadfence();
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
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
        }
        if (lane == 0) p.counters[band] = 0u;
      }
    }
  }

  if (failed) {
    // let this warp's outstanding copies (stages L .. L + kStages - 1) land
    // before the CTA can exit; every wait is bounded again
    for (int LL = L; LL < min(L + kStages, total); ++LL)
      mbar_wait(my_bars + (LL % kStages), (LL / kStages) & 1, p.err);
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
  // raise the kernel's dynamic shared memory limit once (not a stream operation,
  // but kept out of the steady state so launches can be captured in graphs)
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
  gemv_kernel<FMT, MT><<<dim3(pl.ctas_x, pl.S), kWarps * 32, pl.smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

GemvPlan plan_gemv(int fmt, int M, int N, int K, int num_sms) {
  (void)fmt;
  GemvPlan pl;
  pl.mt = M <= 8 ? 1 : (M <= 16 ? 2 : (M <= 32 ? 4 : 8));
  const int NT = (N + 15) / 16;
  const int groups = K / 128;
  const int ring = kWarps * kStages * kStageBytes;
  const int xbudget = kMaxSmem - kHeaderBytes - ring;
  // largest slice (in 128-groups) whose activation image fits
  const int max_groups = (xbudget / M - 16) / 256;
  const int s_min = (groups + max_groups - 1) / max_groups;
  double best = 1e300;
  int best_s = s_min;
  for (int S = s_min; S <= groups && S <= 16; ++S) {
    const int gslice = (groups + S - 1) / S;
    if ((S - 1) * gslice >= groups) continue;  // an empty split
    int ctas = num_sms / S;
    if (ctas < 1) ctas = 1;
    if (ctas > NT) ctas = NT;
    const double bands = static_cast<double>((NT + ctas - 1) / ctas);
    double cost = bands * gslice * (S > 1 ? 1.03 : 1.0);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = S;
    }
  }
  pl.S = best_s;
  const int gslice = (groups + pl.S - 1) / pl.S;
  pl.kslice = gslice * 128;
  int ctas = num_sms / pl.S;
  if (ctas < 1) ctas = 1;
  if (ctas > NT) ctas = NT;
  pl.ctas_x = ctas;
  pl.smem = kHeaderBytes + ring + M * ((pl.kslice / 64) * 128 + 16);
  return pl;
}

size_t gemv_workspace_floats(const GemvPlan& p, int M, int N) {
  return p.S > 1 ? static_cast<size_t>(p.S) * M * ((N + 15) / 16 * 16) : 0;
}

size_t gemv_counters(const GemvPlan& p, int N) { return p.S > 1 ? (N + 15) / 16 : 0; }

cudaError_t launch_gemv(const GemvPlan& p, const GemmArgs& a, cudaStream_t st) {
  if (a.fmt == 0) {
    switch (p.mt) {
      case 1: return launch_t<0, 1>(p, a, st);
      case 2: return launch_t<0, 2>(p, a, st);
      case 4: return launch_t<0, 4>(p, a, st);
      default: return launch_t<0, 8>(p, a, st);
    }
  }
  switch (p.mt) {
    case 1: return launch_t<1, 1>(p, a, st);
    case 2: return launch_t<1, 2>(p, a, st);
    case 4: return launch_t<1, 4>(p, a, st);
    default: return launch_t<1, 8>(p, a, st);
  }
}

}  // namespace w4
