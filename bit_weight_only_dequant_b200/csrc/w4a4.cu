// W4A4 NVFP4: the activations quantised to NVFP4 as well (model card
// "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX", table "Release highlights":
// W4A4 NVFP4, group size 16).  The pages name only the format; the reading
// taken (the plainest one consistent with the weight side of the format):
//
//   g_x = fp32(amax |x|) / fp32(6 * 448)        one fp32 scale per tensor
//                                               (1.0 for an all-zero x)
//   s   = RNE_e4m3(amax_block / (6 * g_x))      one E4M3 scale per row and
//                                               16 consecutive k, saturating
//                                               at 448
//   q   = RNE_e2m1(x / (e4m3(s) * g_x))         E2M1 codes, ties to the even
//                                               code, saturating at +-6
//
// every product and division in fp32 with round-to-nearest (no contraction),
// so the codes and scales are decided exactly as a reference that follows the
// same steps in fp32 decides them.  The rounding onto E4M3 and E2M1 is done
// with explicit comparisons and integer arithmetic, not with the hardware
// conversions, so that every tie and saturation rule is the one stated here.
//
// The quantised activation x_hat = e2m1(q) * e4m3(s) * g_x: e2m1 * e4m3 has
// at most 6 significant bits and lies in [2^-10, 2688], so it is exact in
// BF16 and FP16; the product with g_x is left to the matmul, whose per-tensor
// scale becomes g_w * g_x.  Two matmuls consume the quantiser's outputs: the
// block-scaled tensor-core kernel (bs.cu), which takes the codes two per byte
// and the scales in tensor-memory atoms, and the NVFP4 W4A16 paths of this
// library, which take the block-scaled values as BF16.
#include "bs.h"
#include "common.cuh"
#include "kernels.h"

namespace w4 {

namespace {

// Largest |x| of the tensor as the fp32 bits of a BF16 value (magnitude bits
// compared as integers, which order like the values).  amax_bits is zero on
// entry: the quantiser kernel of the previous call cleared it.  Launched with
// programmatic dependent launch: x may come from the previous kernel.
__global__ void __launch_bounds__(256) act_amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                       long long n8, unsigned* amax_bits,
                                                       int late_trigger) {
  // late_trigger: dependents start only once every kernel ahead of this one
  // has finished (the block-scaled matmul relies on it to load its weights
  // early); otherwise at once
  if (!late_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (late_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint4* v = reinterpret_cast<const uint4*>(x);
  uint32_t mx = 0u;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const uint4 c = __ldg(v + i);
    const uint32_t w[4] = {c.x & 0x7FFF7FFFu, c.y & 0x7FFF7FFFu, c.z & 0x7FFF7FFFu,
                           c.w & 0x7FFF7FFFu};
#pragma unroll
    for (int j = 0; j < 4; ++j) mx = max(mx, max(w[j] & 0xFFFFu, w[j] >> 16));
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, mx << 16);
}

// RNE onto E4M3 of a non-negative, finite fp32 value, saturating at 448
// (0x7E); the value 480 that rounding could reach is not finite in E4M3.
__device__ __forceinline__ uint32_t rne_e4m3(float t) {
  if (!(t > 0.f)) return 0u;
  if (t >= 448.f) return 0x7Eu;
  if (t < 0.015625f) {                               // below 2^-6: quantum 2^-9
    // t * 2^9 is exact; rintf rounds half to even; the result 8 is the
    // smallest normal 2^-6, whose code is also 8
    return (uint32_t)rintf(t * 512.f);
  }
  int e;
  const float m = frexpf(t, &e);                     // t = m 2^e, m in [0.5, 1)
  // 4 significant bits: mantissa steps of 2^(e-4)
  uint32_t r = (uint32_t)rintf(ldexpf(m, 4));        // 8 .. 16, exact scaling
  if (r == 16u) {
    r = 8u;
    ++e;
  }
  // value = r 2^(e-4) = (1 + (r-8)/8) 2^(e-1): exponent field e - 1 + 7
  const uint32_t code = ((uint32_t)(e + 6) << 3) | (r - 8u);
  return code > 0x7Eu ? 0x7Eu : code;
}

// RNE onto E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the code
// whose mantissa bit is 0, saturating at 6; the sign goes to bit 3 (negative
// zero included).  The thresholds are the midpoints between neighbours, each
// tie going to the even side.
__device__ __forceinline__ uint32_t rne_e2m1(float v) {
  const float a = fabsf(v);
  const uint32_t mag = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                       (a >= 3.5f) + (a > 5.f);
  return mag | (signbit(v) ? 8u : 0u);
}

__device__ __forceinline__ float e2m1_mag(uint32_t c) {
  const uint32_t m = c & 7u;
  return m < 2 ? 0.5f * m : ldexpf(1.f + 0.5f * (m & 1u), (int)(m >> 1) - 1);
}

__device__ __forceinline__ float e4m3_val(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e == 0 ? ldexpf((float)m, -9) : ldexpf(1.f + m * 0.125f, (int)e - 7);
}

__device__ __forceinline__ float global_scale(unsigned amax_bits) {
  const float amax = __uint_as_float(amax_bits);
  return amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f;   // 6 * 448 = 2688 exactly
}

// Outputs of the quantiser, each optional.  codes: one per byte [M][K];
// scales: E4M3 [M][K/16]; xq: the block-scaled values e2m1 * e4m3 as BF16
// [M][K]; xc / xsf: the block-scaled tensor-core operand layouts (codes two
// per byte [M][K/2], scale atoms per chunk of `rows` rows, layout_bs.h).
struct QuantOut {
  uint8_t* codes;
  uint8_t* scales;
  __nv_bfloat16* xq;
  uint8_t* xc;
  uint8_t* xsf;
  int rows;
};

// Quantise the 16-block b (row b / (K/16)).
__device__ __forceinline__ void quantize_block(const __nv_bfloat16* __restrict__ x, long long b,
                                               long long nblk, int K, float g, const QuantOut& o) {
  uint8_t* codes = o.codes;
  uint8_t* scales = o.scales;
  __nv_bfloat16* xq = o.xq;
  if (b >= nblk) return;
  const uint4* src = reinterpret_cast<const uint4*>(x) + 2 * b;   // the block's 16 values
  const uint4 c0 = __ldg(src), c1 = __ldg(src + 1);
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  float v[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
  float amax_b = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) amax_b = fmaxf(amax_b, fabsf(v[j]));
  const float t = __fdiv_rn(amax_b, __fmul_rn(6.f, g));
  const uint32_t s8 = rne_e4m3(t);
  const float sv = e4m3_val(s8);
  const float step = __fmul_rn(sv, g);
  uint32_t q[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) q[j] = step > 0.f ? rne_e2m1(__fdiv_rn(v[j], step)) : 0u;
  if (codes) {
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      pk[j] = q[4 * j] | (q[4 * j + 1] << 8) | (q[4 * j + 2] << 16) | (q[4 * j + 3] << 24);
    *reinterpret_cast<uint4*>(codes + 16 * b) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  if (scales) scales[b] = (uint8_t)s8;
  if (o.xc) {
    uint32_t pk[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) pk[j >> 3] |= q[j] << (4 * (j & 7));
    *reinterpret_cast<uint2*>(o.xc + 8 * b) = make_uint2(pk[0], pk[1]);
  }
  if (o.xsf) {
    const long long kblk = K >> 4;
    const long long row = b / kblk;
    const long long blk = b - row * kblk;
    const long long c = row / o.rows;
    o.xsf[bs_scale_offset(c, (int)(row - c * o.rows), blk, K)] = (uint8_t)s8;
  }
  if (xq) {
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // e2m1 * e4m3: at most 6 significant bits, exact in fp32 and in BF16
      const float lo = (q[2 * j] & 8u ? -1.f : 1.f) * e2m1_mag(q[2 * j]) * sv;
      const float hi = (q[2 * j + 1] & 8u ? -1.f : 1.f) * e2m1_mag(q[2 * j + 1]) * sv;
      __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
      o[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    uint4* dst = reinterpret_cast<uint4*>(xq) + 2 * b;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// One thread per (row, 16-block).  Thread 0 also writes g_x and, if g_w is
// given, g_w * g_x (fp32, one rounding): the matmul's per-tensor scale.
// Launched behind act_amax_kernel with programmatic dependent launch; the
// last CTA to finish clears amax_bits[0] and its arrival counter
// amax_bits[1] for the next call.
__global__ void __launch_bounds__(256)
    act_quant_kernel(const __nv_bfloat16* __restrict__ x, int M, int K, unsigned* amax_bits,
                     const float* __restrict__ g_w, const QuantOut o, float* g_x_out,
                     float* g_eff_out, int late_trigger) {
  // late_trigger: dependents start only once every kernel ahead of this one
  // has finished (the block-scaled matmul relies on it to load its weights
  // early); otherwise at once
  if (!late_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (late_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const float g = global_scale(*reinterpret_cast<volatile unsigned*>(amax_bits));
  const long long nblk = (long long)M * (K >> 4);
  const long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (b == 0) {
    if (g_x_out) *g_x_out = g;
    if (g_eff_out) *g_eff_out = g_w ? __fmul_rn(__ldg(g_w), g) : g;
  }
  quantize_block(x, b, nblk, K, g, o);
  // every thread of this CTA has read amax_bits: the last CTA clears it
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    unsigned* done = amax_bits + 1;
    if (atomicAdd(done, 1u) == gridDim.x - 1) {
      amax_bits[0] = 0u;
      *done = 0u;
    }
  }
}

// Small activation tensors (at most kSmallBlocks 16-blocks): one CTA finds
// amax|x| with a block reduction and quantises every block itself, so the
// call is one launch instead of two and touches no amax word.
constexpr int kSmallThreads = 1024;
constexpr long long kSmallBlocks = kSmallThreads / 2;

__global__ void __launch_bounds__(kSmallThreads)
    act_quant_small_kernel(const __nv_bfloat16* __restrict__ x, int M, int K,
                           const float* __restrict__ g_w, const QuantOut o, float* g_x_out,
                           float* g_eff_out, int late_trigger) {
  // late_trigger: dependents start only once every kernel ahead of this one
  // has finished (the block-scaled matmul relies on it to load its weights
  // early); otherwise at once
  if (!late_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (late_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ uint32_t red[kSmallThreads / 32];
  const long long n8 = (long long)M * K / 8, nblk = (long long)M * (K >> 4);
  const uint4* v = reinterpret_cast<const uint4*>(x);
  uint32_t mx = 0u;
  for (long long i = threadIdx.x; i < n8; i += kSmallThreads) {
    const uint4 c = __ldg(v + i);
    const uint32_t w[4] = {c.x & 0x7FFF7FFFu, c.y & 0x7FFF7FFFu, c.z & 0x7FFF7FFFu,
                           c.w & 0x7FFF7FFFu};
#pragma unroll
    for (int j = 0; j < 4; ++j) mx = max(mx, max(w[j] & 0xFFFFu, w[j] >> 16));
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    mx = __reduce_max_sync(0xffffffffu, red[threadIdx.x]);
    if (threadIdx.x == 0) red[0] = mx;
  }
  __syncthreads();
  const float g = global_scale(red[0] << 16);
  if (threadIdx.x == 0) {
    if (g_x_out) *g_x_out = g;
    if (g_eff_out) *g_eff_out = g_w ? __fmul_rn(__ldg(g_w), g) : g;
  }
  for (long long b = threadIdx.x; b < nblk; b += kSmallThreads) quantize_block(x, b, nblk, K, g, o);
}

}  // namespace

namespace {

cudaError_t launch_quant(int M, int K, const void* x, unsigned* amax_bits, const float* g_w,
                         const QuantOut& o, float* g_x, float* g_eff, int late_trigger,
                         cudaStream_t st) {
  // amax_bits[0..1] are zero between calls (zeroed once when the scratch is
  // allocated, cleared again by the last quantiser CTA of every call)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((long long)M * (K / 16) <= kSmallBlocks) {
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(kSmallThreads, 1, 1);
    return cudaLaunchKernelEx(&cfg, act_quant_small_kernel, static_cast<const __nv_bfloat16*>(x),
                              M, K, g_w, o, g_x, g_eff, late_trigger);
  }
  const long long n8 = (long long)M * K / 8;
  cfg.gridDim = dim3((unsigned)min(1184ll, (n8 + 255) / 256), 1, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, act_amax_kernel, static_cast<const __nv_bfloat16*>(x),
                                     n8, amax_bits, late_trigger);
  if (e != cudaSuccess) return e;
  const long long nblk = (long long)M * (K / 16);
  cfg.gridDim = dim3((unsigned)((nblk + 255) / 256), 1, 1);
  return cudaLaunchKernelEx(&cfg, act_quant_kernel, static_cast<const __nv_bfloat16*>(x), M, K,
                            amax_bits, g_w, o, g_x, g_eff, late_trigger);
}

}  // namespace

cudaError_t launch_act_quant(int M, int K, const void* x, unsigned* amax_bits, const float* g_w,
                             void* codes, void* scales, void* xq, float* g_x, float* g_eff,
                             cudaStream_t st) {
  QuantOut o;
  o.codes = static_cast<uint8_t*>(codes);
  o.scales = static_cast<uint8_t*>(scales);
  o.xq = static_cast<__nv_bfloat16*>(xq);
  o.xc = nullptr;
  o.xsf = nullptr;
  o.rows = 1;
  return launch_quant(M, K, x, amax_bits, g_w, o, g_x, g_eff, 0, st);
}

cudaError_t launch_act_quant_bs(int M, int K, int rows, const void* x, unsigned* amax_bits,
                                const float* g_w, void* xc, void* xsf, float* g_x, float* g_eff,
                                cudaStream_t st) {
  QuantOut o;
  o.codes = nullptr;
  o.scales = nullptr;
  o.xq = nullptr;
  o.xc = static_cast<uint8_t*>(xc);
  o.xsf = static_cast<uint8_t*>(xsf);
  o.rows = rows;
  // the block-scaled matmul loads its weights before its own wait while the
  // activations fit one 16-row MMA tile (bs.cu): start it only after the wait
  return launch_quant(M, K, x, amax_bits, g_w, o, g_x, g_eff, rows <= 16 ? 1 : 0, st);
}

}  // namespace w4
