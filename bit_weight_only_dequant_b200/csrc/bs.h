// W4A4 NVFP4 on the block-scaled tensor cores: planner, launchers and the
// activation quantiser's block-scaled outputs (declarations).
#pragma once

#include <cuda_runtime.h>

#include "layout_bs.h"

namespace w4 {

constexpr int kBsStageK = 256;       // k per pipeline stage (128 bytes of codes per row)

struct BsPlan {
  int tiles;        // 128-row weight tiles
  int chunks;       // activation chunks (at most 128 rows each)
  int rows;         // activation rows per chunk
  int mpad;         // rows padded to the MMA N (a multiple of 16)
  int S;            // K splits
  int sps;          // stages (256 k) per split
  int units;        // tiles x chunks x splits
  int grid;         // persistent CTAs
  int nstages;      // shared-memory pipeline stages
  int stage_bytes;  // bytes of one stage
  int smem;         // dynamic shared memory bytes
};

BsPlan plan_bs(int M, int N, int K, int num_sms);
size_t bs_workspace_floats(const BsPlan& p, int M);

// xc: activation codes [M][K/2]; xsf: activation scale atoms per chunk;
// g: device fp32 g_w * g_x; y: [M][N] BF16; ws: split-K partials.
cudaError_t launch_bs(const BsPlan& p, int M, int N, int K, const void* w, const void* sfw,
                      const void* xc, const void* xsf, const float* g, void* y, float* ws,
                      unsigned* err, cudaStream_t st);

// The activation quantiser writing the block-scaled operand layouts: codes
// [M][K/2], scale atoms per chunk of `rows` rows, g_x and g_w * g_x.
cudaError_t launch_act_quant_bs(int M, int K, int rows, const void* x, unsigned* amax_bits,
                                const float* g_w, void* xc, void* xsf, float* g_x, float* g_eff,
                                cudaStream_t st);

cudaError_t launch_pack_bs(int N, int K, const void* codes, const void* scales, void* w, void* s,
                           cudaStream_t st);
int pack_host_bs(int N, int K, const void* codes, const void* scales, void* w, void* s);
int unpack_host_bs(int N, int K, const void* w, const void* s, void* codes, void* scales);

}  // namespace w4
