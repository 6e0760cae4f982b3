// Bit-exact dequantisation of the packed weights into a BF16 [N][K] matrix.
//
// INT4 (forum post "Qwen3.8-27B on single DGX Spark ...", section "Quality"):
//   W = RNE_bf16(q * s); q * s has at most 12 significant bits, so the fp32
//   product is exact and cvt.rn.bf16.f32 is the only rounding.
// NVFP4 (model card "Qwen3.8 27B - NVFP4 for veloGB10", "Specifications"):
//   W = RNE_bf16(e2m1 * e4m3 * g); e2m1 * e4m3 is exact in fp32, times the
//   fp32 g it needs up to 30 bits, so the product is formed in fp64 (exact)
//   and rounded once: fp64 -> fp32 toward zero with a sticky bit (round to
//   odd, 16 spare bits) followed by fp32 -> bf16 to nearest even gives the
//   correctly rounded BF16 value, subnormal range included.
// FP8-E4M3 (weight-only FP8 of the attention linears, guide "Qwen3.8-27B on
//   DGX Spark (GB10)", section "The right stack for Spark"): W = RNE_bf16(e4m3
//   * g) with one fp32 g per tensor, rounded the same way.
#include "common.cuh"
#include "kernels.h"

namespace w4 {

namespace {

__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t mag = c & 7u;
  const float v = mag < 2 ? 0.5f * mag : ldexpf(1.f + 0.5f * (mag & 1u), (int)(mag >> 1) - 1);
  return (c & 8u) ? -v : v;
}

__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  const float v = e == 0 ? ldexpf((float)m, -9) : ldexpf(1.f + m * 0.125f, (int)e - 7);
  return (b & 0x80u) ? -v : v;
}

__device__ __forceinline__ __nv_bfloat16 round_product_bf16(float p, float g) {
  const double d = (double)p * (double)g;  // exact
  float f = __double2float_rz(d);
  if ((double)f != d) f = __uint_as_float(__float_as_uint(f) | 1u);  // round to odd
  return __float2bfloat16_rn(f);
}

template <int FMT>
__global__ void dequant_kernel(int N, int K, const uint8_t* __restrict__ w,
                               const uint8_t* __restrict__ s, const float* __restrict__ gptr,
                               __nv_bfloat16* __restrict__ out) {
  const int KB = K >> 6;
  const long long NT = (N + 15) / 16;
  const long long total = NT * KB * 32;  // one thread per lane chunk of a tile
  const float g = FMT == 1 ? __ldg(gptr) : 1.f;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int lane = (int)(idx & 31);
    const long long tile = idx >> 5;
    const long long nt = tile / KB;
    const int kb = (int)(tile - nt * KB);
    const int gq = lane >> 2, t = lane & 3;
    const uint4 wv = *reinterpret_cast<const uint4*>(w + tile * kTileBytes + lane * 16);
    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const long long n = nt * 16 + gq + 8 * hrow;
      if (n >= N) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k0 = kb * 64 + j * 16 + 4 * t;
        float vals[4];
        if (FMT == 0) {
          const uint16_t sb = *reinterpret_cast<const uint16_t*>(
              s + int4_scale_offset(n, k0 / kInt4Group, K));
          const float sv = __uint_as_float((uint32_t)sb << 16);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int pair = hrow + 2 * (e >> 1), second = e & 1;
            const int nib = pair + 4 * second;
            const int u = (int)((wd[j] >> (4 * nib)) & 15u);
            vals[e] = (float)(u - 8) * sv;  // exact
          }
          __nv_bfloat16 o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) o[e] = __float2bfloat16_rn(vals[e]);
          *reinterpret_cast<uint2*>(out + n * (long long)K + k0) = *reinterpret_cast<uint2*>(o);
        } else {
          const uint8_t sb = s[nvfp4_scale_offset(n, k0 / kNvfp4Group, K)];
          const float sv = e4m3_value(sb);
          __nv_bfloat16 o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int pair = hrow + 2 * (e >> 1), second = e & 1;
            const int nib = 2 * pair + second;
            const uint32_t c = (wd[j] >> (4 * nib)) & 15u;
            o[e] = round_product_bf16(e2m1_value(c) * sv, g);  // e2m1 * e4m3 exact in fp32
          }
          *reinterpret_cast<uint2*>(out + n * (long long)K + k0) = *reinterpret_cast<uint2*>(o);
        }
      }
    }
  }
}

__global__ void dequant_fp8_kernel(int N, int K, const uint8_t* __restrict__ w,
                                   const float* __restrict__ gptr, __nv_bfloat16* __restrict__ out) {
  const int KT = K >> 5;
  const long long NT = (N + 15) / 16;
  const long long total = NT * KT * 32;
  const float g = __ldg(gptr);
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int lane = (int)(idx & 31);
    const long long tile = idx >> 5;
    const long long nt = tile / KT;
    const int kt = (int)(tile - nt * KT);
    const int gq = lane >> 2, t = lane & 3;
    const uint4 wv = *reinterpret_cast<const uint4*>(w + tile * kTileBytes + lane * 16);
    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int hrow = 0; hrow < 2; ++hrow) {
      const long long n = nt * 16 + gq + 8 * hrow;
      if (n >= N) continue;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int k0 = kt * 32 + j * 16 + 4 * t;
        __nv_bfloat16 o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pair = hrow + 2 * (e >> 1), second = e & 1;
          const uint32_t b = (wd[2 * j + (pair >> 1)] >> (8 * (2 * (pair & 1) + second))) & 0xFFu;
          o[e] = round_product_bf16(e4m3_value(b), g);
        }
        *reinterpret_cast<uint2*>(out + n * (long long)K + k0) = *reinterpret_cast<uint2*>(o);
      }
    }
  }
}

}  // namespace

cudaError_t launch_dequant(int fmt, int N, int K, const void* w, const void* s, const float* g,
                           void* out, cudaStream_t st) {
  const long long total = (long long)((N + 15) / 16) * (K / 64) * 32 * (fmt == kFmtFp8 ? 2 : 1);
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (fmt == kFmtFp8)
    dequant_fp8_kernel<<<(unsigned)blocks, 256, 0, st>>>(N, K, (const uint8_t*)w, g,
                                                         (__nv_bfloat16*)out);
  else if (fmt == 0)
    dequant_kernel<0><<<(unsigned)blocks, 256, 0, st>>>(N, K, (const uint8_t*)w, (const uint8_t*)s,
                                                         g, (__nv_bfloat16*)out);
  else
    dequant_kernel<1><<<(unsigned)blocks, 256, 0, st>>>(N, K, (const uint8_t*)w, (const uint8_t*)s,
                                                         g, (__nv_bfloat16*)out);
  return cudaGetLastError();
}

}  // namespace w4
