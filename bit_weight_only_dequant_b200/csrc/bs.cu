// W4A4 NVFP4 on the block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4),
// sm_100a.
//
// With the activations quantised to NVFP4 as well (model card
// "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX", table "Release highlights":
// W4A4 NVFP4, group size 16), both operands of the matmul are E2M1 codes with
// one E4M3 scale per 16 k: the operand format of the block-scaled MMA with
// 16-element scale blocks.  The tensor cores read the packed codes from
// shared memory and the scales from tensor memory, so no instruction of this
// kernel touches a weight; it only streams bytes, and at decode and verify
// row counts its time is the weight bytes over HBM bandwidth.
//
// Structure (one persistent CTA per SM, 6 warps; a unit of work is a
// 128-row weight tile x an activation chunk of at most 128 rows x a K split,
// a pipeline stage is 256 k):
//  * warp 0, one lane (producer): per stage a 2-D TMA load of the weight tile
//    (128 rows x 128 bytes, 128-byte swizzle), one of the activation codes
//    (Mpad rows; rows past M read as zero), and two 1-D bulk copies of 2 KB,
//    the stage's four scale atoms of each operand, all completing on the
//    stage's mbarrier.
//  * warp 1 (MMA, one elected lane): per stage, eight tcgen05.cp 32x128b
//    (the scale atoms into tensor memory, replicated over the four lane
//    quadrants, two stage buffers), then four MMAs of K = 64 (M = 128 weight
//    rows, N = Mpad activation rows, fp32 D in tensor memory); commits free
//    the stage and, at the end of a unit, hand D to the epilogue.
//  * warps 2-5 (epilogue, one lane quadrant each): tcgen05.ld of D, times
//    g_w * g_x, BF16 stores; with K split, fp32 partials that a second kernel
//    (programmatic dependent launch) adds in split order.
// Tensor memory (256 columns): D in [0, 128) -- two buffers of 64 columns
// while Mpad <= 64, so the next unit's MMAs overlap the epilogue -- then the
// scale buffers.  Every mbarrier wait is bounded; a timeout raises the device
// error word and the CTA drains its copies and MMAs and frees tensor memory.
// Launched with programmatic dependent launch right behind the library's own
// activation quantiser.  While the activations fit one 16-row MMA tile the
// quantiser lets dependents start only after its own griddepcontrol.wait: by
// the time this kernel starts every kernel ahead of the quantiser has
// finished, so the weights and their scales are final and the producer loads
// them at once (overlapping the quantiser); only the activation codes and
// scales, which the quantiser writes, wait for griddepcontrol.wait.  With
// more rows (a longer quantiser, which the early weight stream would slow,
// measured) the CTA only prefetches its first weight stages into L2 before
// the wait.
#include <atomic>

#include "bs.h"
#include "common.cuh"
#include "tcgen05.cuh"

namespace w4 {

namespace {

constexpr int kBsThreads = 192;
constexpr int kBsMaxStages = 8;
constexpr int kBsTmemCols = 256;
constexpr int kBsSfaCol = 128;                      // two 16-column buffers each
constexpr int kBsSfbCol = 160;
constexpr int kBsABytes = kBsTileRows * 128;        // weight codes of a stage
constexpr int kBsSfBytes = 4 * kBsAtomBytes;        // one operand's scale atoms of a stage
constexpr int kBsMaxSmem = 227 * 1024;
constexpr int kBsBarBytes = 256;

struct BsParams {
  const uint8_t* sfa;      // weight scale atoms [tiles][K/64]
  const uint8_t* sfb;      // activation scale atoms [chunks][K/64]
  const float* g;          // g_w * g_x
  __nv_bfloat16* y;
  float* ws;               // split-K partials [S][M][Npad]
  unsigned* err;
  int M, N, K, KB64, T;    // T: stages (256 k) along K, the last one half full when K % 256 = 128
  int chunks, rows, mpad, S, sps, units, nstages, stage_bytes, Npad;
};

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory descriptor of one 512-byte scale atom for tcgen05.cp: K-major,
// no swizzle, 32 rows of 16 bytes, i.e. four 8-row core matrices 128 bytes
// apart (stride offset); one core matrix along k (leading offset unused).
__device__ __forceinline__ uint64_t atom_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1u << 46;                 // descriptor version (sm_100); layout 0 = no swizzle
  return d;
}

// 32 rows x 128 bits from shared memory into tensor memory lanes 0-31 (four
// 32-bit columns), copied to each of the four lane quadrants.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[tmem] (+)= (A . sfa) (B . sfb)^T, E2M1 operands from shared memory, E4M3
// scales (one per 16 k) from tensor memory, fp32 D; one CTA.
__device__ __forceinline__ void umma_bs(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], "
      "p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of the block-scaled MMA: A and B E2M1 (format 1 of
// the fp4 kinds), both K-major, N = mpad, M = 128, UE4M3 scales (bit 23 = 0),
// K = 64 (bit 31 = 0), scale-factor byte ids 0.
__host__ __device__ constexpr uint32_t bs_idesc(int mpad) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(mpad >> 3) << 17) |
         ((uint32_t)(kBsTileRows >> 4) << 24);
}

__device__ __forceinline__ void bs_unit(const BsParams& p, int unit, int& tile, int& chunk,
                                        int& split, int& t_lo, int& t_hi) {
  const int per_tile = p.chunks * p.S;
  tile = unit / per_tile;
  const int r = unit - tile * per_tile;
  chunk = r / p.S;
  split = r - chunk * p.S;
  t_lo = split * p.sps;
  t_hi = min(p.T, t_lo + p.sps);
}

__global__ void __launch_bounds__(kBsThreads, 1)
    bs_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
              const BsParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.nstages * p.stage_bytes);
  uint64_t* full = bars;                                 // per stage
  uint64_t* empty = bars + kBsMaxStages;                 // per stage
  uint64_t* dfull = bars + 2 * kBsMaxStages;             // per D buffer
  uint64_t* dfree = dfull + 2;
  uint64_t* drain = dfree + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbuf = p.mpad <= 64 ? 2 : 1;
  const int xbytes = p.mpad * 128;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.nstages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(dfull + i, 1);
      mbar_init(dfree + i, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(kBsTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (lane 0)
    // weights may be loaded before the wait (see above); the quantiser uses
    // the same condition (rows <= 16) for its late trigger
    const bool early = p.rows <= 16;
    if (lane == 0 && !early) {
      if ((int)blockIdx.x < p.units) {
        int tile, chunk, split, t_lo, t_hi;
        bs_unit(p, blockIdx.x, tile, chunk, split, t_lo, t_hi);
        const int t_end = min(t_hi, t_lo + p.nstages);
        for (int t = t_lo; t < t_end; ++t)
          asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                           reinterpret_cast<uint64_t>(&wmap)),
                       "r"(t * 128), "r"(tile * kBsTileRows)
                       : "memory");
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    if (lane == 0) {
      int s = 0;                      // stage of load `it`
      uint32_t u = 0, it = 0;         // times the stages have wrapped; loads issued
      bool ok = true, xr = !early;    // activation loads may be issued (after the wait)
      int np = 0;                     // stages whose activation loads are held back
      int pend_s[kBsMaxStages], pend_t[kBsMaxStages], pend_c[kBsMaxStages];
      auto x_loads = [&](int slot, int t, int chunk) {
        uint8_t* st = smem + slot * p.stage_bytes;
        const uint32_t sf = (uint32_t)min(4, p.KB64 - 4 * t) * kBsAtomBytes;
        tma_load_2d(st + kBsABytes, &xmap, t * 128, chunk * p.rows, full + slot);
        bulk_g2s(smem_u32(st + kBsABytes + xbytes + kBsSfBytes),
                 p.sfb + ((size_t)chunk * p.KB64 + 4 * t) * kBsAtomBytes, sf, full + slot);
      };
      // the quantiser's outputs are complete: issue the held-back loads
      auto x_ready = [&]() {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int i = 0; i < np; ++i) x_loads(pend_s[i], pend_t[i], pend_c[i]);
        np = 0;
        xr = true;
      };
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x) {
        int tile, chunk, split, t_lo, t_hi;
        bs_unit(p, unit, tile, chunk, split, t_lo, t_hi);
        for (int t = t_lo; t < t_hi; ++t) {
          if (u > 0) {
            if (!xr) x_ready();         // a stage is reused only after its MMAs, which need x
            if (!tc_wait(empty + s, (u - 1) & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
          }
          uint8_t* st = smem + s * p.stage_bytes;
          // scale atoms of this stage (2 in a half stage at the end of K);
          // the TMA boxes are always full, k past K reading as zero
          const uint32_t sf = (uint32_t)min(4, p.KB64 - 4 * t) * kBsAtomBytes;
          mbar_arrive_expect_tx(full + s, (uint32_t)(kBsABytes + xbytes) + 2 * sf);
          tma_load_2d(st, &wmap, t * 128, tile * kBsTileRows, full + s);
          bulk_g2s(smem_u32(st + kBsABytes + xbytes),
                   p.sfa + ((size_t)tile * p.KB64 + 4 * t) * kBsAtomBytes, sf, full + s);
          if (xr) {
            x_loads(s, t, chunk);
          } else {
            pend_s[np] = s;
            pend_t[np] = t;
            pend_c[np] = chunk;
            ++np;
          }
          ++it;
          if (++s == p.nstages) {
            s = 0;
            ++u;
          }
        }
      }
      if (!xr) x_ready();
      // every issued copy lands before the CTA may exit
      const uint32_t first = it > (uint32_t)p.nstages ? it - (uint32_t)p.nstages : 0u;
      for (uint32_t k = first; k < it; ++k)
        mbar_wait(full + k % p.nstages, (k / p.nstages) & 1, p.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (whole warp)
    const uint32_t idesc = bs_idesc(p.mpad);
    int s = 0;
    uint32_t par = 0, it = 0, unit_i = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++unit_i) {
      int tile, chunk, split, t_lo, t_hi;
      bs_unit(p, unit, tile, chunk, split, t_lo, t_hi);
      const uint32_t b = nbuf == 2 ? (unit_i & 1u) : 0u;
      const uint32_t uses = nbuf == 2 ? (unit_i >> 1) : unit_i;
      if (uses > 0) {
        if (!warp_wait(dfree + b, (uses - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
      }
      const uint32_t d = tmem + b * 64;
      for (int t = t_lo; t < t_hi; ++t, ++it) {
        if (!warp_wait(full + s, par, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint8_t* st = smem + s * p.stage_bytes;
        const uint64_t adesc = sw128_desc(smem_u32(st));
        const uint64_t bdesc = sw128_desc(smem_u32(st + kBsABytes));
        const uint32_t sa = smem_u32(st + kBsABytes + xbytes), sb = sa + kBsSfBytes;
        const uint32_t sfa = tmem + kBsSfaCol + 16 * (it & 1u);
        const uint32_t sfb = tmem + kBsSfbCol + 16 * (it & 1u);
        const int nk = min(4, p.KB64 - 4 * t);           // MMAs of K = 64 in this stage
        if (elect_one()) {
          for (int kk = 0; kk < nk; ++kk) {
            tmem_cp_32x128b_x4(sfa + 4 * kk, atom_desc(sa + kk * kBsAtomBytes));
            tmem_cp_32x128b_x4(sfb + 4 * kk, atom_desc(sb + kk * kBsAtomBytes));
          }
          // K = 64 (32 bytes of codes) per MMA: the descriptors advance 2 x 16 bytes
          for (int kk = 0; kk < nk; ++kk)
            umma_bs(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, sfa + 4 * kk, sfb + 4 * kk,
                    (t > t_lo || kk > 0) ? 1u : 0u);
          umma_commit(empty + s);
        }
        __syncwarp();
        if (++s == p.nstages) {
          s = 0;
          par ^= 1u;
        }
      }
      if (ok) {
        if (elect_one()) umma_commit(dfull + b);
        __syncwarp();
      }
    }
    // every MMA is issued: the split-K reduction grid may be scheduled
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // drain: all issued copies and MMAs complete before tensor memory is released
    if (elect_one()) {
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2-5)
    // g and y may be read or written by the previous kernel on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int q = warp & 3;                         // this warp's tensor-memory lane quadrant
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    uint32_t unit_i = 0;
    for (int unit = blockIdx.x; unit < p.units; unit += gridDim.x, ++unit_i) {
      int tile, chunk, split, t_lo, t_hi;
      bs_unit(p, unit, tile, chunk, split, t_lo, t_hi);
      const uint32_t b = nbuf == 2 ? (unit_i & 1u) : 0u;
      const uint32_t uses = nbuf == 2 ? (unit_i >> 1) : unit_i;
      if (!warp_wait(dfull + b, uses & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const int n = tile * kBsTileRows + 32 * q + lane;
      const int xrow = chunk * p.rows;
      const int mlim = min(p.rows, p.M - xrow);
      const float gm = p.S == 1 ? __ldg(p.g) : 1.f;
#pragma unroll 1
      for (int c0 = 0; c0 < p.mpad; c0 += 16) {
        float v[16];
        tmem_ld_32x32b<16>(tmem + lane_off + b * 64 + c0, v);
        tmem_wait_ld();
        if (n < p.N) {
          if (p.S == 1) {
            __nv_bfloat16* yp = p.y + (size_t)(xrow + c0) * p.N + n;
#pragma unroll
            for (int c = 0; c < 16; ++c)
              if (c0 + c < mlim) yp[(size_t)c * p.N] = __float2bfloat16_rn(v[c] * gm);
          } else {
            float* wp = p.ws + ((size_t)split * p.M + xrow + c0) * p.Npad + n;
#pragma unroll
            for (int c = 0; c < 16; ++c)
              if (c0 + c < mlim) __stcg(wp + (size_t)c * p.Npad, v[c]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dfree + b);
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kBsTmemCols));
  }
}

// y[m][n] = BF16(g * sum over splits, in split order, of the fp32 partials
// [S][M][Npad]); four columns per thread, launched behind the main kernel
// with programmatic dependent launch.
__global__ void __launch_bounds__(256)
    bs_splitk_reduce(const float* __restrict__ ws, int S, int M, int N, int Npad,
                     const float* __restrict__ g, __nv_bfloat16* __restrict__ y) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int m = blockIdx.y;
  const int n0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (n0 >= N) return;
  const float* src = ws + (size_t)m * Npad + n0;
  const size_t sstride = (size_t)M * Npad;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  for (int sp = 0; sp < S; ++sp) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(src + sp * sstride));
    a[0] += v.x;
    a[1] += v.y;
    a[2] += v.z;
    a[3] += v.w;
  }
  const float gm = __ldg(g);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (n0 + j < N) y[(size_t)m * N + n0 + j] = __float2bfloat16_rn(a[j] * gm);
}

// 2-D tensor map over a byte matrix [rows][row_bytes] with 128-byte swizzled
// boxes of 128 bytes x box_rows (rows past the end read as zero).
bool make_u8_map(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

// Splits K so that the units (128-row tiles x chunks x splits) fill the SMs:
// the estimated time is waves x (stages per unit + one stage of per-unit
// cost), plus about four stages for the reduction launch when K is split.
BsPlan plan_bs(int M, int N, int K, int num_sms) {
  BsPlan pl{};
  if (M < 1 || N < 1 || K < 128 || K % 128 != 0 || num_sms < 1) return pl;
  pl.tiles = (int)bs_tiles(N);
  pl.chunks = (M + 127) / 128;
  pl.rows = (M + pl.chunks - 1) / pl.chunks;
  pl.mpad = ((pl.rows + 15) / 16) * 16;
  const int T = (K + kBsStageK - 1) / kBsStageK;
  const long long base = (long long)pl.tiles * pl.chunks;
  double best = 1e300;
  for (int S = 1; S <= T && S <= 64; ++S) {
    const int sps = (T + S - 1) / S;
    if ((T + sps - 1) / sps != S) continue;       // every split holds at least one stage
    const long long units = base * S;
    const long long waves = (units + num_sms - 1) / num_sms;
    const double cost = (double)waves * (sps + 1.0) + (S > 1 ? 4.0 : 0.0);
    if (cost < best - 1e-9) {
      best = cost;
      pl.S = S;
      pl.sps = sps;
    }
  }
  pl.units = (int)(base * pl.S);
  pl.grid = pl.units < num_sms ? pl.units : num_sms;
  pl.stage_bytes = kBsABytes + pl.mpad * 128 + 2 * kBsSfBytes;
  pl.nstages = (kBsMaxSmem - 1024 - kBsBarBytes) / pl.stage_bytes;
  if (pl.nstages > kBsMaxStages) pl.nstages = kBsMaxStages;
  pl.smem = pl.nstages * pl.stage_bytes + kBsBarBytes + 1024;
  return pl;
}

size_t bs_workspace_floats(const BsPlan& p, int M) {
  return p.S > 1 ? (size_t)p.S * M * p.tiles * kBsTileRows : 0;
}

cudaError_t launch_bs(const BsPlan& pl, int M, int N, int K, const void* w, const void* sfw,
                      const void* xc, const void* xsf, const float* g, void* y, float* ws,
                      unsigned* err, cudaStream_t st) {
  if (pl.S < 1 || pl.nstages < 2) return cudaErrorInvalidValue;
  CUtensorMap wmap, xmap;
  if (!make_u8_map(&wmap, w, N, K / 2, kBsTileRows) || !make_u8_map(&xmap, xc, M, K / 2, pl.mpad))
    return cudaErrorInvalidValue;
  BsParams p;
  p.sfa = static_cast<const uint8_t*>(sfw);
  p.sfb = static_cast<const uint8_t*>(xsf);
  p.g = g;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ws = ws;
  p.err = err;
  p.M = M;
  p.N = N;
  p.K = K;
  p.KB64 = K / 64;
  p.T = (K + kBsStageK - 1) / kBsStageK;
  p.chunks = pl.chunks;
  p.rows = pl.rows;
  p.mpad = pl.mpad;
  p.S = pl.S;
  p.sps = pl.sps;
  p.units = pl.units;
  p.nstages = pl.nstages;
  p.stage_bytes = pl.stage_bytes;
  p.Npad = pl.tiles * kBsTileRows;
  // the dynamic shared memory limit, raised once per device (atomic: host
  // threads may race here; the attribute call is idempotent)
  static std::atomic<int> smem_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem_set[dev].load(std::memory_order_acquire) < pl.smem) {
    const cudaError_t e =
        cudaFuncSetAttribute(bs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return e;
    int cur = smem_set[dev].load(std::memory_order_relaxed);
    while (cur < pl.smem && !smem_set[dev].compare_exchange_weak(cur, pl.smem)) {
    }
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.grid, 1, 1);
  cfg.blockDim = dim3(kBsThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)pl.smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, bs_kernel, wmap, xmap, p);
  if (e != cudaSuccess || pl.S == 1) return e;
  cfg.gridDim = dim3((unsigned)((N + 1023) / 1024), (unsigned)M, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, bs_splitk_reduce, static_cast<const float*>(ws), pl.S, M, N,
                            p.Npad, g, static_cast<__nv_bfloat16*>(y));
}

}  // namespace w4
