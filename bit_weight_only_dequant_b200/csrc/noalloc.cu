// w4a16_gemm_noalloc: the split-K GEMV for callers that cannot allocate
// device memory.
//
// Who needs it: applications that reserve all device memory up front for
// their own allocator or pool (serving engines that hand every byte to
// weights and KV cache) and forbid any later cudaMalloc, including the hidden
// one that w4a16_gemm makes the first time a stream needs split-K workspace;
// and latency-critical code that must not call cudaMalloc in its steady state,
// since an allocation can synchronise the device and stall every stream.
//
// The scratch lives in one file-scope __device__ array of kScratchBytes that
// every GPU which loads this library keeps until the process exits.  Host code
// only ever sees a host-side stand-in for the array's name; the device address
// is fetched once per device with cudaGetSymbolAddress (with that device
// current) and passed to the kernel.  Every call shares the array: calls whose
// GPU work overlaps (two streams, or two host threads on one device) race, and
// the array keeps whatever the last call left there, so each call clears the
// part that must start at zero (the split-K arrival counters) with a
// stream-ordered memset.  The GEMV has no bounded waits, so a call cannot
// time out; the first 256 bytes of the array are reserved.
#include <mutex>

#include "../../include/w4a16.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;      // 8 MiB
constexpr size_t kStatusBytes = 256;            // reserved, keeps the counters aligned
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct NoAllocDevice {
  bool ready = false;
  bool sm100 = false;
  int num_sms = 0;
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch
};

std::mutex g_na_mu;
NoAllocDevice g_na_dev[64];

// Once per device, with that device current: check the architecture,
// resolve the device address of the scratch array and set the launch
// attributes of every GEMV kernel variant this entry point can launch, so that
// later calls (of any shape) only launch.  Allocates nothing.
int noalloc_setup(NoAllocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
  if (dev < 0 || dev >= 64) return W4A16_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_na_mu);
  NoAllocDevice& d = g_na_dev[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return W4A16_ERR_CUDA;
    d.sm100 = prop.major == 10 && prop.minor == 0;
    d.num_sms = prop.multiProcessorCount;
    if (d.sm100) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return W4A16_ERR_CUDA;
      d.base = static_cast<unsigned char*>(ptr);
      if (w4::gemv_prepare_all(0) != cudaSuccess) return W4A16_ERR_CUDA;
    }
    d.ready = true;
  }
  if (!d.sm100) return W4A16_ERR_DEVICE;
  *out = &d;
  return W4A16_OK;
}

}  // namespace

extern "C" int w4a16_gemm_noalloc(int fmt, int M, int N, int K, const void* x_bf16,
                                  const void* packed_w, const void* packed_scales,
                                  const float* global_scale, void* y_bf16, void* stream) {
  if (fmt != W4A16_FMT_INT4_G128 && fmt != W4A16_FMT_NVFP4_G16 && fmt != W4A16_FMT_FP8_E4M3)
    return W4A16_ERR_ARG;
  if (N < 1 || K < 128 || K % 128 != 0) return W4A16_ERR_SHAPE;
  if ((long long)((N + 15) / 16) * (K / 64) >= (1ll << 31) / 64) return W4A16_ERR_SHAPE;
  if (M < 1 || M > W4A16_GEMV_MAX_M) return W4A16_ERR_SHAPE;
  const bool scaled = fmt != W4A16_FMT_FP8_E4M3;   // FP8 has no packed scales
  if (!x_bf16 || !packed_w || !y_bf16 || (scaled && !packed_scales)) return W4A16_ERR_ARG;
  if ((fmt != W4A16_FMT_INT4_G128) != (global_scale != nullptr)) return W4A16_ERR_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(packed_w) |
                        (scaled ? reinterpret_cast<uintptr_t>(packed_scales) : 0) |
                        reinterpret_cast<uintptr_t>(y_bf16);
  if (mis & 15u) return W4A16_ERR_ALIGN;

  NoAllocDevice* d = nullptr;
  int r = noalloc_setup(&d);
  if (r != W4A16_OK) return r;

  const w4::GemvPlan pl = w4::plan_gemv(fmt, M, N, K, d->num_sms);
  if (pl.S == 0) return W4A16_ERR_SHAPE;
  const size_t counters = w4::gemv_counters(pl, N);
  const size_t floats = w4::gemv_workspace_floats(pl, M, N);
  const size_t counter_bytes = (counters * sizeof(unsigned) + 255) / 256 * 256;
  if (kStatusBytes + counter_bytes + floats * sizeof(float) > kScratchBytes)
    return W4A16_ERR_SCRATCH;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = reinterpret_cast<unsigned*>(d->base);
  unsigned* cnt = reinterpret_cast<unsigned*>(d->base + kStatusBytes);
  float* part = reinterpret_cast<float*>(d->base + kStatusBytes + counter_bytes);
  if (cudaMemsetAsync(d->base, 0, kStatusBytes + counter_bytes, st) != cudaSuccess)
    return W4A16_ERR_CUDA;

  w4::GemmArgs a;
  a.fmt = fmt;
  a.M = M;
  a.N = N;
  a.K = K;
  a.x = x_bf16;
  a.w = packed_w;
  a.s = packed_scales;
  a.g = global_scale;
  a.y = y_bf16;
  a.ws = floats > 0 ? part : nullptr;
  a.counters = counters > 0 ? cnt : nullptr;
  a.err = status;
  return w4::launch_gemv(pl, a, st) == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA;
}
