// Internal launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace w4 {

struct GemmArgs {
  int fmt;
  int M, N, K;
  const void* x;        // [M][K] bf16
  const void* w;        // packed weights
  const void* s;        // packed scales
  const float* g;       // nvfp4 per-tensor scale (device) or null
  void* y;              // [M][N] bf16
  float* ws;            // split-K partials (fp32), may be null when no split is used
  unsigned* counters;   // per 16-row band arrival counters (zero between calls)
  unsigned* err;        // device error word
  int fuse = 0;         // 1: fused gate/up layer, N = 2I weight rows (gate first),
                        //    y = [M][I] holds SiLU(gate) * up
};

// ---------------------------------------------------------------- GEMV (M <= 16)

struct GemvPlan {
  int S;         // K splits
  int kslice;    // K elements per split (multiple of 128)
  int ctas_x;    // CTAs per split
  int mt;        // 8-row activation tiles (1: M <= 8, 2: M <= 16)
  int wn, wk;    // warps per CTA as (bands in flight) x (K pieces per band)
  int depth;     // shared-memory ring stages (128-groups in flight) per warp
  int ngp;       // 128-groups per warp piece, padded to a multiple of depth
  int smem;      // dynamic shared memory bytes
};

GemvPlan plan_gemv(int fmt, int M, int N, int K, int num_sms, int fuse = 0);
// Bytes of fp32 workspace and number of counters the plan needs.
size_t gemv_workspace_floats(const GemvPlan& p, int M, int N);
size_t gemv_counters(const GemvPlan& p, int N);
cudaError_t launch_gemv(const GemvPlan& p, const GemmArgs& a, cudaStream_t st);
// Set the launch attributes of every GEMV kernel variant (plain or fused) on
// the current device, so that no later launch has to.
cudaError_t gemv_prepare_all(int fuse);

// ---------------------------------------------------------------- tensor-core path (tcgen05)

// Row chunking: M rows run as ceil(M / kTcMaxRows) chunks of `rows` rows
// each (the last one may be shorter), as units of one launch.
constexpr int kTcMaxRows = 128;

struct TcPlan {
  int chunks;    // activation chunks
  int rows;      // activation rows per chunk (M split evenly into <= kTcMaxRows)
  int mpad;      // rows padded to the MMA N (a multiple of 16, at most 128)
  int S;         // K splits
  int kbs;       // 64-blocks per split
  int units;     // 256-row tiles x chunks x splits
  int grid;      // persistent CTAs
  int smem;      // dynamic shared memory bytes
};

TcPlan plan_tc(int fmt, int M, int N, int K, int num_sms, int fuse = 0);
size_t tc_workspace_floats(const TcPlan& p, int M, int N);
size_t tc_counters(const TcPlan& p, int N);
size_t tc_x_f16_bytes(int fmt, int M, int K);   // NVFP4: FP16 copy of x + row multipliers
cudaError_t launch_tc(const TcPlan& p, const GemmArgs& a, void* xf16_scratch, cudaStream_t st);
// Diagnostics: a bounded mbarrier wait that is made to run out (see capi.cu).
cudaError_t launch_wait_timeout_selftest(unsigned* err, int* out, cudaStream_t st);

// ---------------------------------------------------------------- W4A4: activation quantiser

// x [M][K] BF16 -> NVFP4 (codes, E4M3 block scales, fp32 g_x); every output
// optional.  amax_bits: one device word of scratch.  xq: the block-scaled
// values e2m1 * e4m3 as BF16 [M][K]; g_eff: g_w * g_x (g_w may be null: g_x).
cudaError_t launch_act_quant(int M, int K, const void* x, unsigned* amax_bits, const float* g_w,
                             void* codes, void* scales, void* xq, float* g_x, float* g_eff,
                             cudaStream_t st);

// ---------------------------------------------------------------- dequant export / packer

cudaError_t launch_dequant(int fmt, int N, int K, const void* w, const void* s, const float* g,
                           void* out, cudaStream_t st);
cudaError_t launch_pack(int fmt, int N, int K, const void* codes, const void* scales, void* w,
                        void* s, cudaStream_t st);
// Host packer / unpacker; 0 on success, -1 on an out-of-range code or scale.
int pack_host(int fmt, int N, int K, const void* codes, const void* scales, void* w, void* s);
int unpack_host(int fmt, int N, int K, const void* w, const void* s, void* codes, void* scales);

}  // namespace w4
