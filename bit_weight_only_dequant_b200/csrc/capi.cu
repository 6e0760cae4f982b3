// C ABI of the library (include/w4a16.h): argument validation, per-device
// state, the row-count dispatcher and the split-K workspace.
#include <map>
#include <mutex>
#include <utility>

#include "../../include/w4a16.h"
#include "bs.h"
#include "common.cuh"
#include "kernels.h"

namespace {

struct DeviceState {
  bool checked = false;
  bool ok = false;        // sm_100
  int dev = 0;
  int num_sms = 0;
  unsigned* err = nullptr;  // device error word
};

struct Workspace {
  void* base = nullptr;   // [counters (uint32)] [partials (fp32)] [scratch bytes]
  size_t counters = 0;
  size_t floats = 0;
  size_t bytes = 0;
};

std::mutex g_mu;
std::map<int, DeviceState> g_dev;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

// Plans depend only on (format, M, N, K) and the SM count: computed once per
// shape and device (a decode step calls the same few shapes every token).
struct PlanKey {
  int dev, fmt, M, N, K, fuse;
  bool operator<(const PlanKey& o) const {
    if (dev != o.dev) return dev < o.dev;
    if (fuse != o.fuse) return fuse < o.fuse;
    if (fmt != o.fmt) return fmt < o.fmt;
    if (M != o.M) return M < o.M;
    if (N != o.N) return N < o.N;
    return K < o.K;
  }
};
std::map<PlanKey, w4::GemvPlan> g_gemv_plans;
std::map<PlanKey, w4::TcPlan> g_tc_plans;

w4::GemvPlan cached_gemv_plan(int dev, int fmt, int M, int N, int K, int num_sms, int fuse) {
  const PlanKey key{dev, fmt, M, N, K, fuse};
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_gemv_plans.find(key);
  if (it != g_gemv_plans.end()) return it->second;
  const w4::GemvPlan pl = w4::plan_gemv(fmt, M, N, K, num_sms, fuse);
  if (g_gemv_plans.size() < 4096) g_gemv_plans.emplace(key, pl);
  return pl;
}

w4::TcPlan cached_tc_plan(int dev, int fmt, int M, int N, int K, int num_sms, int fuse) {
  const PlanKey key{dev, fmt, M, N, K, fuse};
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_tc_plans.find(key);
  if (it != g_tc_plans.end()) return it->second;
  const w4::TcPlan pl = w4::plan_tc(fmt, M, N, K, num_sms, fuse);
  if (g_tc_plans.size() < 4096) g_tc_plans.emplace(key, pl);
  return pl;
}

int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.checked) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return W4A16_ERR_CUDA;
    d.ok = prop.major == 10 && prop.minor == 0;
    d.dev = dev;
    d.num_sms = prop.multiProcessorCount;
    if (d.ok) {
      if (cudaMalloc(&d.err, sizeof(unsigned)) != cudaSuccess) return W4A16_ERR_NOMEM;
      if (cudaMemset(d.err, 0, sizeof(unsigned)) != cudaSuccess) return W4A16_ERR_CUDA;
    }
    d.checked = true;
  }
  if (!d.ok) return W4A16_ERR_DEVICE;
  *out = &d;
  return W4A16_OK;
}

// Workspace of at least (counters, floats, bytes) for the current device and
// `st`.  Grows by reallocation in stream order; counters start (and are left) zero.
int workspace(cudaStream_t st, size_t counters, size_t floats, size_t bytes, unsigned** cnt,
              float** part, void** scratch) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[std::make_pair(dev, st)];
  if (w.base == nullptr || w.counters < counters || w.floats < floats || w.bytes < bytes) {
    size_t nc = counters > w.counters ? counters : w.counters;
    size_t nf = floats > w.floats ? floats : w.floats;
    size_t nb = bytes > w.bytes ? bytes : w.bytes;
    if (nc < 65536) nc = 65536;
    if (nf < (1u << 20)) nf = 1u << 20;
    nc = (nc + 63) / 64 * 64;
    nf = (nf + 63) / 64 * 64;
    nb = (nb + 255) / 256 * 256;
    void* base = nullptr;
    if (cudaMallocAsync(&base, nc * sizeof(unsigned) + nf * sizeof(float) + nb, st) != cudaSuccess)
      return W4A16_ERR_NOMEM;
    if (cudaMemsetAsync(base, 0, nc * sizeof(unsigned), st) != cudaSuccess) return W4A16_ERR_CUDA;
    if (w.base) cudaFreeAsync(w.base, st);
    w.base = base;
    w.counters = nc;
    w.floats = nf;
    w.bytes = nb;
  }
  *cnt = static_cast<unsigned*>(w.base);
  *part = reinterpret_cast<float*>(static_cast<unsigned*>(w.base) + w.counters);
  *scratch = reinterpret_cast<uint8_t*>(*part + w.floats);
  return W4A16_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool has_global_scale(int fmt) { return fmt != W4A16_FMT_INT4_G128; }
bool has_packed_scales(int fmt) { return fmt != W4A16_FMT_FP8_E4M3; }

// allow_bs: the block-scaled W4A4 weight layout (packers, sizes, its matmul)
int check_fmt_shape(int fmt, int N, int K, bool allow_bs = false) {
  if (fmt != W4A16_FMT_INT4_G128 && fmt != W4A16_FMT_NVFP4_G16 && fmt != W4A16_FMT_FP8_E4M3 &&
      !(allow_bs && fmt == W4A16_FMT_NVFP4_BS))
    return W4A16_ERR_ARG;
  if (N < 1 || K < 128 || K % 128 != 0) return W4A16_ERR_SHAPE;
  // packed tensors are addressed with 32-bit tile/scale indices in places
  if ((long long)((N + 15) / 16) * (K / 64) >= (1ll << 31) / 64) return W4A16_ERR_SHAPE;
  return W4A16_OK;
}

// Row-count dispatch: the weight-streaming GEMV while the activations are a
// thin n8 operand, the tcgen05 path once the tensor cores carry real work.
// The crossovers come from back-to-back timings of both paths on the decode
// shapes (B200), the same for int4 and NVFP4 (FP8 follows them): the GEMV wins up to M = 8
// everywhere and at M = 9..16 for the widest layer (N >= 16384: enough
// 16-row bands per SM); the tensor-core path wins for the other layers at
// M >= 9 and everywhere at M > 16.
int choose_path(int fmt, int M, int N, int K) {
  (void)fmt;
  (void)K;
  if (M <= 8) return W4A16_PATH_GEMV;
  if (M <= W4A16_GEMV_MAX_M && N >= 16384) return W4A16_PATH_GEMV;
  return W4A16_PATH_TC;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? W4A16_OK : W4A16_ERR_CUDA; }

// The matmul (fuse = 0) or the fused gate/up layer (fuse = 1, N = 2I rows,
// y = [M][I]) on the chosen path.
int run_gemm(int path, int fmt, int M, int N, int K, const void* x_bf16, const void* packed_w,
             const void* packed_scales, const float* global_scale, void* y_bf16, void* stream,
             int fuse) {
  int r = check_fmt_shape(fmt, N, K);
  if (r != W4A16_OK) return r;
  if (M < 1 || M > W4A16_MAX_M) return W4A16_ERR_SHAPE;
  if (path != W4A16_PATH_AUTO && path != W4A16_PATH_GEMV && path != W4A16_PATH_TC)
    return W4A16_ERR_ARG;
  if (!x_bf16 || !packed_w || !y_bf16) return W4A16_ERR_ARG;
  if (has_packed_scales(fmt) && !packed_scales) return W4A16_ERR_ARG;
  if (has_global_scale(fmt) != (global_scale != nullptr)) return W4A16_ERR_ARG;
  if (!aligned16(x_bf16) || !aligned16(packed_w) || !aligned16(y_bf16) ||
      (has_packed_scales(fmt) && !aligned16(packed_scales)))
    return W4A16_ERR_ALIGN;
  if (path == W4A16_PATH_AUTO) path = choose_path(fmt, M, N, K);
  if (path == W4A16_PATH_GEMV && M > W4A16_GEMV_MAX_M) return W4A16_ERR_SHAPE;
  DeviceState* d = nullptr;
  if ((r = device_state(&d)) != W4A16_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

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
  a.ws = nullptr;
  a.counters = nullptr;
  a.err = d->err;
  a.fuse = fuse;
  void* scratch = nullptr;
  if (path == W4A16_PATH_GEMV) {
    const w4::GemvPlan pl = cached_gemv_plan(d->dev, fmt, M, N, K, d->num_sms, fuse);
    if (pl.S == 0) return W4A16_ERR_SHAPE;
    const size_t nf = w4::gemv_workspace_floats(pl, M, N);
    if (nf > 0) {
      r = workspace(st, w4::gemv_counters(pl, N), nf, 0, &a.counters, &a.ws, &scratch);
      if (r != W4A16_OK) return r;
    }
    return status_of(w4::launch_gemv(pl, a, st));
  }
  const w4::TcPlan pl = cached_tc_plan(d->dev, fmt, M, N, K, d->num_sms, fuse);
  const size_t nf = w4::tc_workspace_floats(pl, M, N);
  const size_t nb = w4::tc_x_f16_bytes(fmt, M, K);
  if (nf > 0 || nb > 0) {
    r = workspace(st, w4::tc_counters(pl, N), nf, nb, &a.counters, &a.ws, &scratch);
    if (r != W4A16_OK) return r;
  }
  return status_of(w4::launch_tc(pl, a, scratch, st));
}

}  // namespace

extern "C" {

size_t w4a16_packed_weight_bytes(int fmt, int N, int K) {
  if (check_fmt_shape(fmt, N, K, true) != W4A16_OK) return 0;
  if (fmt == W4A16_FMT_NVFP4_BS) return (size_t)w4::bs_weight_bytes(N, K);
  return (size_t)w4::weight_bytes(fmt, N, K);
}

size_t w4a16_packed_scale_bytes(int fmt, int N, int K) {
  if (check_fmt_shape(fmt, N, K, true) != W4A16_OK) return 0;
  if (fmt == W4A16_FMT_NVFP4_BS) return (size_t)w4::bs_scale_bytes(N, K);
  return (size_t)w4::scale_bytes(fmt, N, K);
}

int w4a16_pack_host(int fmt, int N, int K, const void* codes, const void* scales, void* packed_w,
                    void* packed_scales) {
  const int r = check_fmt_shape(fmt, N, K, true);
  if (r != W4A16_OK) return r;
  if (!codes || !packed_w || (has_packed_scales(fmt) && (!scales || !packed_scales)))
    return W4A16_ERR_ARG;
  if (fmt == W4A16_FMT_NVFP4_BS)
    return w4::pack_host_bs(N, K, codes, scales, packed_w, packed_scales) == 0 ? W4A16_OK
                                                                              : W4A16_ERR_ARG;
  return w4::pack_host(fmt, N, K, codes, scales, packed_w, packed_scales) == 0 ? W4A16_OK
                                                                               : W4A16_ERR_ARG;
}

int w4a16_unpack_host(int fmt, int N, int K, const void* packed_w, const void* packed_scales,
                      void* codes, void* scales) {
  const int r = check_fmt_shape(fmt, N, K, true);
  if (r != W4A16_OK) return r;
  if (!codes || !packed_w || (has_packed_scales(fmt) && (!scales || !packed_scales)))
    return W4A16_ERR_ARG;
  if (fmt == W4A16_FMT_NVFP4_BS)
    return w4::unpack_host_bs(N, K, packed_w, packed_scales, codes, scales) == 0 ? W4A16_OK
                                                                                : W4A16_ERR_ARG;
  return w4::unpack_host(fmt, N, K, packed_w, packed_scales, codes, scales) == 0 ? W4A16_OK
                                                                                 : W4A16_ERR_ARG;
}

int w4a16_pack(int fmt, int N, int K, const void* codes, const void* scales, void* packed_w,
               void* packed_scales, void* stream) {
  int r = check_fmt_shape(fmt, N, K, true);
  if (r != W4A16_OK) return r;
  if (!codes || !packed_w || (has_packed_scales(fmt) && (!scales || !packed_scales)))
    return W4A16_ERR_ARG;
  if (!aligned16(codes) || !aligned16(packed_w) ||
      (has_packed_scales(fmt) && (!aligned16(scales) || !aligned16(packed_scales))))
    return W4A16_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((r = device_state(&d)) != W4A16_OK) return r;
  if (fmt == W4A16_FMT_NVFP4_BS)
    return status_of(w4::launch_pack_bs(N, K, codes, scales, packed_w, packed_scales,
                                        static_cast<cudaStream_t>(stream)));
  return status_of(w4::launch_pack(fmt, N, K, codes, scales, packed_w, packed_scales,
                                   static_cast<cudaStream_t>(stream)));
}

int w4a16_dequant(int fmt, int N, int K, const void* packed_w, const void* packed_scales,
                  const float* global_scale, void* w_bf16, void* stream) {
  int r = check_fmt_shape(fmt, N, K);
  if (r != W4A16_OK) return r;
  if (!packed_w || !w_bf16 || (has_packed_scales(fmt) && !packed_scales)) return W4A16_ERR_ARG;
  if (has_global_scale(fmt) != (global_scale != nullptr)) return W4A16_ERR_ARG;
  if (!aligned16(packed_w) || !aligned16(w_bf16) ||
      (has_packed_scales(fmt) && !aligned16(packed_scales)))
    return W4A16_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((r = device_state(&d)) != W4A16_OK) return r;
  return status_of(w4::launch_dequant(fmt, N, K, packed_w, packed_scales, global_scale, w_bf16,
                                      static_cast<cudaStream_t>(stream)));
}

// W4A4: scratch of its own per (device, stream) -- [amax word, arrival
// counter, g_eff, pad to 256 B][block-scaled activations BF16 M x K] -- so that the matmul's
// own workspace can grow without freeing memory this call still reads.
std::map<std::pair<int, cudaStream_t>, Workspace> g_w4a4_ws;

int w4a4_scratch(cudaStream_t st, size_t bytes, uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W4A16_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_w4a4_ws[std::make_pair(dev, st)];
  if (w.base == nullptr || w.bytes < bytes) {
    size_t nb = bytes > 2 * w.bytes ? bytes : 2 * w.bytes;
    nb = (nb + 255) / 256 * 256;
    void* base = nullptr;
    if (cudaMallocAsync(&base, nb, st) != cudaSuccess) return W4A16_ERR_NOMEM;
    // the quantiser's amax word and arrival counter start (and are left) zero
    if (cudaMemsetAsync(base, 0, 256, st) != cudaSuccess) return W4A16_ERR_CUDA;
    if (w.base) cudaFreeAsync(w.base, st);
    w.base = base;
    w.bytes = nb;
  }
  *out = static_cast<uint8_t*>(w.base);
  return W4A16_OK;
}

int w4a16_gemm_path(int fmt, int M, int N, int K) {
  const int r = check_fmt_shape(fmt, N, K);
  if (r != W4A16_OK) return r;
  if (M < 1 || M > W4A16_MAX_M) return W4A16_ERR_SHAPE;
  return choose_path(fmt, M, N, K);
}

int w4a16_gemm_ex(int path, int fmt, int M, int N, int K, const void* x_bf16, const void* packed_w,
                  const void* packed_scales, const float* global_scale, void* y_bf16,
                  void* stream) {
  return run_gemm(path, fmt, M, N, K, x_bf16, packed_w, packed_scales, global_scale, y_bf16,
                  stream, 0);
}

int w4a16_gemm_gate_up_silu_ex(int path, int fmt, int M, int I, int K, const void* x_bf16,
                               const void* packed_w, const void* packed_scales,
                               const float* global_scale, void* h_bf16, void* stream) {
  if (I < 16 || I % 16 != 0 || I > (1 << 29)) return W4A16_ERR_SHAPE;
  return run_gemm(path, fmt, M, 2 * I, K, x_bf16, packed_w, packed_scales, global_scale, h_bf16,
                  stream, 1);
}

int w4a16_gemm_gate_up_silu(int fmt, int M, int I, int K, const void* x_bf16,
                            const void* packed_w, const void* packed_scales,
                            const float* global_scale, void* h_bf16, void* stream) {
  return w4a16_gemm_gate_up_silu_ex(W4A16_PATH_AUTO, fmt, M, I, K, x_bf16, packed_w,
                                    packed_scales, global_scale, h_bf16, stream);
}

int w4a16_gemm(int fmt, int M, int N, int K, const void* x_bf16, const void* packed_w,
               const void* packed_scales, const float* global_scale, void* y_bf16, void* stream) {
  return w4a16_gemm_ex(W4A16_PATH_AUTO, fmt, M, N, K, x_bf16, packed_w, packed_scales,
                       global_scale, y_bf16, stream);
}

int w4a16_quantize_act_nvfp4(int M, int K, const void* x_bf16, void* codes, void* scales,
                             float* g_x, void* stream) {
  if (M < 1 || M > W4A16_MAX_M || K < 128 || K % 128 != 0) return W4A16_ERR_SHAPE;
  if (!x_bf16 || !codes || !scales || !g_x) return W4A16_ERR_ARG;
  if (!aligned16(x_bf16) || !aligned16(codes)) return W4A16_ERR_ALIGN;
  DeviceState* d = nullptr;
  int r = device_state(&d);
  if (r != W4A16_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* scratch = nullptr;
  if ((r = w4a4_scratch(st, 256, &scratch)) != W4A16_OK) return r;
  return status_of(w4::launch_act_quant(M, K, x_bf16, reinterpret_cast<unsigned*>(scratch),
                                        nullptr, codes, scales, nullptr, g_x, nullptr, st));
}

int w4a16_gemm_w4a4_ex(int path, int M, int N, int K, const void* x_bf16, const void* packed_w,
                       const void* packed_scales, const float* global_scale_w, void* y_bf16,
                       void* stream) {
  int r = check_fmt_shape(W4A16_FMT_NVFP4_G16, N, K);
  if (r != W4A16_OK) return r;
  if (M < 1 || M > W4A16_MAX_M) return W4A16_ERR_SHAPE;
  if (!x_bf16 || !packed_w || !packed_scales || !global_scale_w || !y_bf16) return W4A16_ERR_ARG;
  if (!aligned16(x_bf16) || !aligned16(packed_w) || !aligned16(packed_scales) || !aligned16(y_bf16))
    return W4A16_ERR_ALIGN;
  if (path != W4A16_PATH_AUTO && path != W4A16_PATH_GEMV && path != W4A16_PATH_TC)
    return W4A16_ERR_ARG;
  if (path == W4A16_PATH_GEMV && M > W4A16_GEMV_MAX_M) return W4A16_ERR_SHAPE;
  DeviceState* d = nullptr;
  if ((r = device_state(&d)) != W4A16_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* scratch = nullptr;
  if ((r = w4a4_scratch(st, 256 + (size_t)M * K * 2, &scratch)) != W4A16_OK) return r;
  unsigned* amax = reinterpret_cast<unsigned*>(scratch);
  float* g_eff = reinterpret_cast<float*>(scratch + 8);
  void* xq = scratch + 256;
  cudaError_t e = w4::launch_act_quant(M, K, x_bf16, amax, global_scale_w, nullptr, nullptr, xq,
                                       nullptr, g_eff, st);
  if (e != cudaSuccess) return W4A16_ERR_CUDA;
  // the block-scaled activations are exact BF16 values; the NVFP4 matmul on
  // them with the per-tensor scale g_w * g_x is the W4A4 product
  return run_gemm(path, W4A16_FMT_NVFP4_G16, M, N, K, xq, packed_w, packed_scales, g_eff, y_bf16,
                  stream, 0);
}

int w4a16_gemm_w4a4(int M, int N, int K, const void* x_bf16, const void* packed_w,
                    const void* packed_scales, const float* global_scale_w, void* y_bf16,
                    void* stream) {
  return w4a16_gemm_w4a4_ex(W4A16_PATH_AUTO, M, N, K, x_bf16, packed_w, packed_scales,
                            global_scale_w, y_bf16, stream);
}

// Block-scaled W4A4: the quantiser writes the activation operands in the
// tensor cores' layout (codes [M][K/2], scale atoms per chunk), then the
// block-scaled matmul streams both.  Scratch: [amax word, arrival counter,
// g_eff, pad to 256 B][codes M x K/2][scale atoms chunks x K/64 x 512].
int w4a16_gemm_w4a4_bs(int M, int N, int K, const void* x_bf16, const void* packed_w,
                       const void* packed_sf, const float* global_scale_w, void* y_bf16,
                       void* stream) {
  int r = check_fmt_shape(W4A16_FMT_NVFP4_BS, N, K, true);
  if (r != W4A16_OK) return r;
  if (M < 1 || M > W4A16_MAX_M) return W4A16_ERR_SHAPE;
  if (!x_bf16 || !packed_w || !packed_sf || !global_scale_w || !y_bf16) return W4A16_ERR_ARG;
  if (!aligned16(x_bf16) || !aligned16(packed_w) || !aligned16(packed_sf) || !aligned16(y_bf16))
    return W4A16_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((r = device_state(&d)) != W4A16_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const w4::BsPlan pl = w4::plan_bs(M, N, K, d->num_sms);
  if (pl.S == 0) return W4A16_ERR_SHAPE;
  const size_t xc_bytes = ((size_t)M * K / 2 + 255) / 256 * 256;
  const size_t xsf_bytes = (size_t)pl.chunks * (K / 64) * w4::kBsAtomBytes;
  uint8_t* scratch = nullptr;
  if ((r = w4a4_scratch(st, 256 + xc_bytes + xsf_bytes, &scratch)) != W4A16_OK) return r;
  unsigned* amax = reinterpret_cast<unsigned*>(scratch);
  float* g_eff = reinterpret_cast<float*>(scratch + 8);
  uint8_t* xc = scratch + 256;
  uint8_t* xsf = xc + xc_bytes;
  float* ws = nullptr;
  const size_t nf = w4::bs_workspace_floats(pl, M);
  if (nf > 0) {
    unsigned* cnt = nullptr;
    void* unused = nullptr;
    if ((r = workspace(st, 0, nf, 0, &cnt, &ws, &unused)) != W4A16_OK) return r;
  }
  // the matmul must be the very next launch after the quantiser: it loads
  // its weights before its dependent-launch wait, relying on the quantiser
  // starting dependents only once everything ahead of it has finished
  cudaError_t e = w4::launch_act_quant_bs(M, K, pl.rows, x_bf16, amax, global_scale_w, xc, xsf,
                                          nullptr, g_eff, st);
  if (e != cudaSuccess) return W4A16_ERR_CUDA;
  return status_of(w4::launch_bs(pl, M, N, K, packed_w, packed_sf, xc, xsf, g_eff, y_bf16, ws,
                                 d->err, st));
}

int w4a16_plan(int path, int fmt, int M, int N, int K, int fuse, int num_sms, int* out,
               int out_len) {
  if (fuse != 0 && fuse != 1) return W4A16_ERR_ARG;
  const int r = check_fmt_shape(fmt, N, K, path == W4A16_PATH_BS);
  if (r != W4A16_OK) return r;
  if (M < 1 || M > W4A16_MAX_M || num_sms < 1 || !out || out_len < 9) return W4A16_ERR_ARG;
  if (path == W4A16_PATH_BS) {
    if (fmt != W4A16_FMT_NVFP4_BS || fuse) return W4A16_ERR_ARG;
    const w4::BsPlan pl = w4::plan_bs(M, N, K, num_sms);
    const int v[9] = {pl.tiles, pl.chunks, pl.rows, pl.mpad, pl.S, pl.sps, pl.units, pl.grid, pl.smem};
    for (int i = 0; i < 9; ++i) out[i] = v[i];
    return pl.S == 0 ? W4A16_ERR_SHAPE : W4A16_PATH_BS;
  }
  if (fmt == W4A16_FMT_NVFP4_BS) return W4A16_ERR_ARG;
  if (fuse && (N % 32 != 0)) return W4A16_ERR_SHAPE;
  if (path == W4A16_PATH_AUTO) path = choose_path(fmt, M, N, K);
  if (path == W4A16_PATH_GEMV) {
    if (M > W4A16_GEMV_MAX_M) return W4A16_ERR_SHAPE;
    const w4::GemvPlan pl = w4::plan_gemv(fmt, M, N, K, num_sms, fuse);
    const int v[9] = {pl.S, pl.kslice, pl.ctas_x, pl.mt, pl.wn, pl.wk, pl.depth, pl.ngp, pl.smem};
    for (int i = 0; i < 9; ++i) out[i] = v[i];
    return pl.S == 0 ? W4A16_ERR_SHAPE : W4A16_PATH_GEMV;
  }
  if (path != W4A16_PATH_TC) return W4A16_ERR_ARG;
  const w4::TcPlan pl = w4::plan_tc(fmt, M, N, K, num_sms, fuse);
  const int v[9] = {pl.chunks, pl.rows, pl.mpad, pl.S, pl.kbs, pl.units, pl.grid, pl.smem, 0};
  for (int i = 0; i < 9; ++i) out[i] = v[i];
  return W4A16_PATH_TC;
}

int w4a16_selftest_wait_timeout(void* stream) {
  DeviceState* d = nullptr;
  int r = device_state(&d);
  if (r != W4A16_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return W4A16_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpy(&h, d->err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return W4A16_ERR_CUDA;
  if (h) return W4A16_ERR_TIMEOUT;   // an earlier timeout is still unreported
  int* out = nullptr;
  if (cudaMalloc(&out, 2 * sizeof(int)) != cudaSuccess) return W4A16_ERR_NOMEM;
  int res[2] = {0, 0};
  cudaError_t e = cudaMemset(out, 0, 2 * sizeof(int));
  if (e == cudaSuccess) e = w4::launch_wait_timeout_selftest(d->err, out, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(res, out, sizeof(res), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&h, d->err, sizeof(unsigned), cudaMemcpyDeviceToHost);
  cudaFree(out);
  if (e != cudaSuccess) return W4A16_ERR_CUDA;
  if (cudaMemset(d->err, 0, sizeof(unsigned)) != cudaSuccess) return W4A16_ERR_CUDA;
  // as designed: both warps gave up and exactly the timeout bit was recorded
  return (res[0] == 1 && res[1] == 1 && h == w4::kErrTimeout) ? W4A16_OK : W4A16_ERR_TIMEOUT;
}

int w4a16_device_status(void* stream) {
  DeviceState* d = nullptr;
  int r = device_state(&d);
  if (r != W4A16_OK) return r;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return W4A16_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpy(&h, d->err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return W4A16_ERR_CUDA;
  if (h) {
    if (cudaMemset(d->err, 0, sizeof(unsigned)) != cudaSuccess) return W4A16_ERR_CUDA;
    return W4A16_ERR_TIMEOUT;
  }
  return W4A16_OK;
}

const char* w4a16_status_string(int status) {
  switch (status) {
    case W4A16_OK: return "W4A16_OK";
    case W4A16_ERR_ARG: return "W4A16_ERR_ARG: bad argument";
    case W4A16_ERR_SHAPE: return "W4A16_ERR_SHAPE: unsupported M, N or K";
    case W4A16_ERR_ALIGN: return "W4A16_ERR_ALIGN: pointer not 16-byte aligned";
    case W4A16_ERR_DEVICE: return "W4A16_ERR_DEVICE: current device is not sm_100";
    case W4A16_ERR_CUDA: return "W4A16_ERR_CUDA: CUDA runtime error";
    case W4A16_ERR_TIMEOUT: return "W4A16_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case W4A16_ERR_NOMEM: return "W4A16_ERR_NOMEM: workspace allocation failed";
    case W4A16_ERR_SCRATCH: return "W4A16_ERR_SCRATCH: problem exceeds the fixed no-alloc scratch";
    default: return "unknown status";
  }
}

int w4a16_version(void) { return 100; }

}  // extern "C"
