// Device twin of the seeded input generator in synth/__init__.py.
//
// It implements the same published definitions (SplitMix64 used counter-style,
// Box-Muller normals, round-to-nearest-even onto BF16 / FP8-E4M3) so that
// inputs too large to draw on the host (a 64-layer sweep holds ~11 GB of
// packed weights) can be drawn on the GPU, element for element equal to the
// host draws.  It holds no arithmetic of the weight-only matmul itself.
#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t mix64_h(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t stream_key(uint64_t seed, uint64_t tensor) {
  const uint64_t a = mix64_h(seed + kGamma);
  return mix64_h(a + tensor * kGamma);
}

__device__ __forceinline__ uint64_t raw64(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * kGamma);
}

__device__ __forceinline__ double unit(uint64_t z) { return ((double)(z >> 11) + 0.5) * 0x1p-53; }

__device__ __forceinline__ double normal(uint64_t key, uint64_t i) {
  const double u1 = unit(raw64(key, 2 * i));
  const double u2 = unit(raw64(key, 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);
}

__device__ __forceinline__ uint16_t to_bf16_bits(double v) {
  double r;
  if (fabs(v) < 0x1p-126) {
    r = ldexp(rint(ldexp(v, 133)), -133);
  } else {
    int e;
    const double m = frexp(v, &e);
    r = ldexp(rint(ldexp(m, 8)), e - 8);
  }
  return (uint16_t)(__float_as_uint((float)r) >> 16);
}

__device__ __forceinline__ uint8_t to_e4m3_byte(double v) {  // v >= 0, finite
  double r;
  if (v < 0x1p-6) {
    r = ldexp(rint(ldexp(v, 9)), -9);
  } else {
    int e;
    const double m = frexp(v, &e);
    r = ldexp(rint(ldexp(m, 4)), e - 4);
  }
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return 0;
  if (r < 0x1p-6) return (uint8_t)ldexp(r, 9);
  int e;
  const double m = frexp(r, &e);  // r = m 2^e, m in [0.5, 1)
  const int field = e - 1 + 7;
  const int mant = (int)(ldexp(m, 4) - 8.0);
  return (uint8_t)((field << 3) | mant);
}

// kind: 0 int4 q (int8), 1 int4 scales (bf16), 2 activations (bf16),
//       3 nvfp4 codes (uint8), 4 nvfp4 scales (e4m3)
__global__ void gen_kernel(int kind, uint64_t key, long long count, void* out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x) {
    switch (kind) {
      case 0:
        static_cast<int8_t*>(out)[i] = (int8_t)((int)(raw64(key, (uint64_t)i) >> 60) - 8);
        break;
      case 1:
        static_cast<uint16_t*>(out)[i] = to_bf16_bits(0.01 * exp(0.25 * normal(key, (uint64_t)i)));
        break;
      case 2:
        static_cast<uint16_t*>(out)[i] = to_bf16_bits(normal(key, (uint64_t)i));
        break;
      case 3:
        static_cast<uint8_t*>(out)[i] = (uint8_t)(raw64(key, (uint64_t)i) >> 60);
        break;
      default:
        static_cast<uint8_t*>(out)[i] = to_e4m3_byte(fabs(normal(key, (uint64_t)i)) * 0.05);
        break;
    }
  }
}

}  // namespace

extern "C" {

// Fills `count` elements (indices 0..count-1 of the stream (seed, tensor_id))
// of the tensor kind described above into the device buffer `out`.
int synth_generate(int kind, unsigned long long seed, int tensor_id, long long count, void* out,
                   void* stream) {
  if (kind < 0 || kind > 4 || count < 0 || (count > 0 && out == nullptr)) return -1;
  if (count == 0) return 0;
  const uint64_t key = stream_key(seed, (uint64_t)tensor_id);
  long long blocks = (count + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  gen_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(kind, key, count, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}
