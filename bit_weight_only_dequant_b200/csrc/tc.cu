// Tensor-core path for speculative-verify and prefill row counts
// (M = 9 .. 8192) on sm_100a.
//
// At M = 64 the matmul does 256 flops per packed weight byte, close to the
// B200 ridge, so the multiply-adds belong on the 5th-generation tensor cores
// (the pages' remark that verifying several drafted tokens in one pass turns
// a bandwidth-bound step into a slightly compute-bound one: blog post "One
// Config Line Made My 27B Model 2.7x Faster", section "The fix").
//
// Structure (one persistent CTA per SM, 18 warps, 256-row x M tiles; the
// unit of work is one 128-group of K, i.e. one group scale):
//  * warps 0-15 (dequant, then epilogue): one 16-row band each.  Every warp
//    streams its band's packed weights and scales through its own ring of
//    shared-memory stages with cp.async (each lane copies and reads back only
//    its own bytes, as in the GEMV), turns its 32 bytes per group into 64
//    scaled operands in registers (int4: q -> BF16 times the BF16 group scale
//    with one rounding, exactly W_deq; NVFP4: e2m1 -> FP16 times the E4M3
//    scale, exact; FP8: e4m3 -> FP16, exact, the per-tensor scale applied in
//    the epilogue) and writes them straight into a tensor-memory A slot with
//    tcgen05.st 16x256b, whose register layout matches the packed pairs.
//    Shared memory never holds dequantised weights.  Fused gate/up layer:
//    the first 128-row half takes 8 gate bands and the second the matching
//    up bands, so the epilogue finds gate and up of a row in one TMEM lane.
//  * warp 16 (producer): lane 0 loads the two SWIZZLE_128B activation boxes
//    of each group with 2-D TMA (rows past M zero-filled) into a ring.
//  * warp 17 (MMA): tcgen05.mma kind::f16, A (weights, 128 rows) from tensor
//    memory, B (activations, K-major SW128) from shared memory, fp32 D
//    (128 lanes x Mpad columns) per 128-row half; 16 MMAs per group, issued
//    by one elected lane of a converged warp.
//  * epilogue: tcgen05.ld of D, BF16 stores, or fp32 split-K partials that a
//    second kernel (all SMs, programmatic dependent launch) sums in split
//    order.
// Tensor memory: D (two 128-row halves of Mpad columns), then A slots of one
// group (2 halves x 64 columns) in the rest of the 512 columns.  Every
// mbarrier wait is bounded and polled by all lanes of the waiting warp; a
// timeout raises the device error word, the CTA drains its copies and MMAs
// and frees tensor memory.  int4 launches use programmatic dependent launch:
// before the previous kernel has finished, the first weight groups are only
// prefetched into L2; everything read into the SM (weights, x) and every
// result is read or written after griddepcontrol.wait.
//
// M > 128 runs as chunks of at most 128 activation rows (the MMA's N); a unit
// of work is (tile, chunk, K split), and the chunks of one tile are adjacent
// units, so their weight reads mostly hit L2.  Beyond M = 128 the tensor
// cores, not HBM, set the time.
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace w4 {

namespace {

constexpr int kDeqWarps = 16;                 // one 16-row band per warp
constexpr int kTcThreads = (kDeqWarps + 2) * 32;
constexpr int kProducerWarp = kDeqWarps;
constexpr int kMmaWarp = kDeqWarps + 1;
constexpr int kTcTileRows = 256;              // 16 bands, two 128-row MMA tiles
constexpr int kWRing = 4;                     // weight stages (groups) per dequant warp
constexpr int kTmemCols = 512;
constexpr int kGroupBytesW = 2 * kTileBytes;  // one band's packed weights per 128-group
constexpr int kMinSmem = 120 * 1024;          // keeps one CTA (and one TMEM owner) per SM
constexpr int kMaxSmem = 227 * 1024;          // dynamic shared memory limit of one CTA

// Weight ring stage: the group's two tiles (each lane's 16 bytes at 16 lane),
// then the scales each lane needs (int4: 4 bytes at 4 lane; NVFP4: 2 x 8 at 16 lane).
// FP8-E4M3: four 512-byte tiles per band-group, no packed scales.
__host__ __device__ constexpr int tc_group_bytes(int fmt) { return fmt == kFmtFp8 ? 4 * kTileBytes : kGroupBytesW; }
__host__ __device__ constexpr int tc_stage_bytes(int fmt) {
  return fmt == kFmtFp8 ? tc_group_bytes(fmt) : kGroupBytesW + (fmt == 0 ? 128 : 512);
}

struct TcParams {
  const uint8_t* w;
  const uint8_t* s;
  const float* g;
  const float* row_mul;    // NVFP4: per-row power-of-two activation scale
  __nv_bfloat16* y;
  float* ws;               // split-K partials [S][M][Npad] (S > 1)
  unsigned* err;
  int M, N, K, KB, NT, tiles, S, gps, units;   // gps: 128-groups per split
  int chunks, rows;        // activation rows run as `chunks` slices of `rows`
  int fuse, I;             // fused gate/up: I output rows, gate bands [0, I/16), up after
};


// ------------------------------------------------------------------ tcgen05 wrappers

__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// D[tmem] (+)= A[tmem] . B[smem desc]^T, kind::f16, one CTA.
__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor: fp32 D, A/B type (0 f16, 1 bf16), both K-major, M=128, N=mpad.
__host__ __device__ constexpr uint32_t make_idesc(int ab_type, int mpad) {
  return (1u << 4) | ((uint32_t)ab_type << 7) | ((uint32_t)ab_type << 10) |
         ((uint32_t)(mpad >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hmul2_f16(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// ------------------------------------------------------------------ the kernel



// Per activation width MPAD (rows of x padded to 16, at most 128 per launch):
// tensor memory holds D (two 128-row halves of MPAD fp32 columns, 64 apart up
// to MPAD = 64) and then as many A slots of one group (2 halves x 64 columns)
// as fit; the activation ring has four stages where they fit in shared memory.
template <int FMT, int MPAD>
struct TcShape {
  static constexpr int kDStride = MPAD <= 64 ? 64 : 128;     // columns between the D halves
  static constexpr int kAColBase = 2 * kDStride;
  static constexpr int kASlots = (kTmemCols - kAColBase) / 128;
  static constexpr int kXStage = 2 * MPAD * 128;             // two 64-k activation boxes
  static constexpr int kWRingBytes = kDeqWarps * kWRing * tc_stage_bytes(FMT);
  // activation stages (groups): as many as fit, up to 8.  Every CTA reads the
  // same activation tile at about the same time, so a load takes thousands
  // of cycles to land (measured); the depth of this ring, not the bytes,
  // sets how fast the MMA warp can be fed.
  static constexpr int kXFit = (kMaxSmem - kWRingBytes - 2048) / kXStage;
  static constexpr int kXRing = kXFit > 8 ? 8 : kXFit;
  static constexpr int kSmemUse = kXRing * kXStage + kWRingBytes + 1024 /* barriers */;
  static constexpr int kSmem = (kSmemUse + 1024 /* align */ > kMinSmem) ? kSmemUse + 1024 : kMinSmem;
  static_assert(kSmem <= kMaxSmem, "stage rings exceed shared memory");
  static_assert(kXRing >= 3, "activation ring");
  static_assert(2 * kXRing + 2 * kASlots + 4 <= 128, "barrier area");
  static_assert(kASlots >= 2 && kAColBase + kASlots * 128 <= kTmemCols, "tensor memory layout");
  static_assert(MPAD % 16 == 0 && MPAD <= kTcMaxRows, "MMA N");
};

__device__ __forceinline__ void cpa16(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cpa8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A unit is (256-row tile, activation chunk, K split); units of one tile are
// adjacent, so CTAs working at the same time share its weights in L2.
// Returns the tile, the chunk, the split and its K range in 128-groups.
__device__ __forceinline__ void unit_range(const TcParams& p, int unit, int& tile, int& chunk,
                                           int& split, int& g_lo, int& g_hi) {
  const int per_tile = p.chunks * p.S;
  tile = unit / per_tile;
  const int r = unit - tile * per_tile;
  chunk = r / p.S;
  split = r - chunk * p.S;
  const int G = p.K >> 7;
  g_lo = split * p.gps;
  g_hi = min(G, g_lo + p.gps);
}

template <int FMT, int MPAD>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap xmap, const TcParams p) {
  using Sh = TcShape<FMT, MPAD>;
  constexpr int kSB = tc_stage_bytes(FMT);
  constexpr int kXRing = Sh::kXRing, kASlots = Sh::kASlots, kAColBase = Sh::kAColBase;
  constexpr int kDStride = Sh::kDStride;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* Xs = smem;                                    // kXRing x (2 boxes of MPAD x 128 B), SW128
  uint8_t* Wr = Xs + kXRing * Sh::kXStage;               // dequant warps' weight rings
  uint64_t* bars = reinterpret_cast<uint64_t*>(Wr + Sh::kWRingBytes);
  uint64_t* xfull = bars;                                // kXRing
  uint64_t* xfree = bars + kXRing;                       // kXRing
  uint64_t* afull = bars + 2 * kXRing;                   // kASlots
  uint64_t* afree = afull + kASlots;                     // kASlots
  uint64_t* dfull = afree + kASlots;
  uint64_t* dfree = dfull + 1;
  uint64_t* drain = dfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXRing; ++i) {
      mbar_init(xfull + i, 1);
      mbar_init(xfree + i, 1);
    }
    for (int i = 0; i < kASlots; ++i) {
      mbar_init(afull + i, kDeqWarps);
      mbar_init(afree + i, 1);
    }
    mbar_init(dfull, 1);
    mbar_init(dfree, kDeqWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- activations (lane 0)
    // launched with programmatic dependent launch: x (and its FP16 copy) may
    // come from the previous kernel on the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t it = 0;
    bool ok = true;
    if (lane == 0) {
      int s = 0;                      // ring stage of group `it`
      uint32_t u = 0;                 // times the ring has wrapped (it / kXRing)
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x) {
        int tile, chunk, split, g_lo, g_hi;
        unit_range(p, unit, tile, chunk, split, g_lo, g_hi);
        const int xrow = chunk * p.rows;
        for (int gi = g_lo; gi < g_hi; ++gi, ++it, s = s + 1 == kXRing ? 0 : s + 1,
                 u += s == 0 ? 1u : 0u) {
          if (u > 0 && !tc_wait(xfree + s, (u - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(xfull + s, Sh::kXStage);
          uint8_t* dst = Xs + s * Sh::kXStage;
          tma_load_2d(dst, &xmap, gi * 128, xrow, xfull + s);
          tma_load_2d(dst + MPAD * 128, &xmap, gi * 128 + 64, xrow, xfull + s);
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      const uint32_t issued = it;
      for (uint32_t k = issued > kXRing ? issued - kXRing : 0; k < issued; ++k)
        mbar_wait(xfull + k % kXRing, (k / kXRing) & 1, p.err);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer (whole warp)
    constexpr uint32_t idesc = make_idesc(FMT == 0 ? 1 : 0, MPAD);
    uint32_t it = 0, unit_i = 0;
    int x_slot = 0, a_slot = 0;       // stage / slot of group `it`
    uint32_t x_par = 0, a_par = 0;    // their phase parity
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++unit_i) {
      int tile, chunk, split, g_lo, g_hi;
      unit_range(p, unit, tile, chunk, split, g_lo, g_hi);
      (void)tile;
      (void)chunk;
      if (unit_i > 0) {
        if (!warp_wait(dfree, (unit_i - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
      }
      for (int gi = g_lo; gi < g_hi; ++gi, ++it) {
        const int xs_ = x_slot, sl = a_slot;
        if (!warp_wait(xfull + xs_, x_par, abort_flag, p.err) ||
            !warp_wait(afull + sl, a_par, abort_flag, p.err)) {
          ok = false;
          break;
        }
        // the next group's stage / slot and phase parity (no division)
        if (++x_slot == kXRing) {
          x_slot = 0;
          x_par ^= 1u;
        }
        if (++a_slot == kASlots) {
          a_slot = 0;
          a_par ^= 1u;
        }
        tc_fence_after();
        const uint64_t b0 = sw128_desc(smem_u32(Xs + xs_ * Sh::kXStage));
        const uint32_t a0 = tmem + kAColBase + sl * 128;
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(tmem + h * kDStride, a0 + h * 64 + kk * 8,
                      b0 + (uint64_t)(((kk >> 2) * MPAD * 128) >> 4) + (uint64_t)((kk & 3) * 2),
                      idesc, (gi > g_lo || kk > 0) ? 1u : 0u);
          umma_commit(afree + sl);
          umma_commit(xfree + xs_);
        }
        __syncwarp();
      }
      if (ok) {
        if (elect_one()) umma_commit(dfull);
        __syncwarp();
      }
    }
    // every MMA is issued: the split-K reduction grid may be scheduled
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // drain: all issued MMAs complete before tensor memory is released
    if (elect_one()) {
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- dequant + epilogue
    const int q = warp & 3, h = (warp >> 2) & 1, bp = warp >> 3;
    const int band = h * 8 + 2 * q + bp;                // 16-row band of the 256-row tile
    const int g = lane >> 2;
    const uint32_t lane_base = (uint32_t)(32 * q + 16 * bp) << 16;
    const uint64_t pol = policy_evict_first();
    const int G = p.K >> 7;
    constexpr int kSStep = FMT == 0 ? 32 : FMT == 1 ? 128 : 0;   // one band's scale bytes per group
    constexpr int kGB = tc_group_bytes(FMT);             // one band's weight bytes per group
    constexpr int kTPG = kGB / kTileBytes;

    // copy cursor over this warp's groups: (unit, group) in the CTA's order
    uint8_t* ring = Wr + warp * kWRing * kSB;
    const uint32_t ring_s = smem_u32(ring) + lane * 16;
    int c_unit = blockIdx.x, c_gi = 0, c_hi = 0, c_nb = 0;
    bool c_valid = false;
    const uint8_t* cw = nullptr;
    const uint8_t* cs = nullptr;
    auto c_start = [&]() {
      if (c_unit < p.units) {
        int tile, chunk, split, g_lo;
        unit_range(p, c_unit, tile, chunk, split, g_lo, c_hi);
        c_gi = g_lo;
        // weight band: tile x 16 bands, or (fused) 8 gate bands in half 0
        // and the matching up bands, I/16 further, in half 1
        c_nb = p.fuse ? (h ? p.I >> 4 : 0) + tile * 8 + (band & 7) : tile * 16 + band;
        c_valid = p.fuse ? tile * 8 + (band & 7) < (p.I >> 4) : c_nb < p.NT;
        const int nb = min(c_nb, p.NT - 1);
        cw = p.w + ((size_t)nb * p.KB * (kTPG / 2) + kTPG * g_lo) * kTileBytes + lane * 16;
        cs = FMT == 0   ? p.s + ((size_t)nb * G + g_lo) * 32 + g * 4
             : FMT == 1 ? p.s + ((size_t)nb * p.KB + 2 * g_lo) * 64 + g * 8
                        : p.s;
      }
    };
    c_start();
    uint32_t c_it = 0;
    auto copy_next = [&]() {                            // one group -> stage c_it % kWRing
      if (c_unit < p.units) {
        if (c_valid) {
          const uint32_t d = ring_s + (c_it % kWRing) * kSB;
#pragma unroll
          for (int i = 0; i < kTPG; ++i) cpa16(d + i * kTileBytes, cw + i * kTileBytes, pol);
          if (FMT == 0) {
            cpa4(d + kGroupBytesW - lane * 12, cs);       // scale slot: lane * 4
          } else if (FMT == 1) {
            cpa8(d + kGroupBytesW, cs);
            cpa8(d + kGroupBytesW + 8, cs + 64);
          }
        }
        cw += kGB;
        cs += kSStep;
        if (++c_gi == c_hi) {
          c_unit += gridDim.x;
          c_start();
        }
      }
      cpa_commit();
      ++c_it;
    };
    // Before the previous kernel on the stream has finished, only an L2 hint
    // for the first groups of this band (the weights may have been written by
    // that kernel, a packer for instance); every read into the SM comes after
    // griddepcontrol.wait.
    if (lane == 0 && c_unit < p.units && c_valid) {
      const int n0 = min(kWRing, c_hi - c_gi);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(cw), "r"((uint32_t)n0 * kGB)
                   : "memory");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
    for (int k = 0; k < kWRing; ++k) copy_next();

    uint32_t it = 0, unit_i = 0;
    int sl = 0;                       // tensor-memory slot of group `it`
    uint32_t ua = 0;                  // times the slots have wrapped (it / kASlots)
    const uint32_t a_base = tmem + lane_base + kAColBase + h * 64;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++unit_i) {
      int tile, chunk, split, g_lo, g_hi;
      unit_range(p, unit, tile, chunk, split, g_lo, g_hi);
      const bool real_band = p.fuse ? tile * 8 + (band & 7) < (p.I >> 4) : tile * 16 + band < p.NT;
      for (int gi = g_lo; gi < g_hi; ++gi, ++it) {
        cpa_wait<kWRing - 1>();                          // this lane's bytes of group `it`
        const uint8_t* st = ring + (it % kWRing) * kSB;
        uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0, w2 = w0, w3 = w0;
        uint32_t sv0 = 0, sv1 = 0, sv2 = 0, sv3 = 0;
        if (real_band) {
          w0 = *reinterpret_cast<const uint4*>(st + lane * 16);
          w1 = *reinterpret_cast<const uint4*>(st + kTileBytes + lane * 16);
          if (FMT == kFmtFp8) {
            w2 = *reinterpret_cast<const uint4*>(st + 2 * kTileBytes + lane * 16);
            w3 = *reinterpret_cast<const uint4*>(st + 3 * kTileBytes + lane * 16);
          } else if (FMT == 0) {
            sv0 = *reinterpret_cast<const uint32_t*>(st + kGroupBytesW + lane * 4);
          } else {
            const uint4 sv = *reinterpret_cast<const uint4*>(st + kGroupBytesW + lane * 16);
            sv0 = sv.x; sv1 = sv.y; sv2 = sv.z; sv3 = sv.w;
          }
        }
        __syncwarp();
        copy_next();                                     // refill the stage just read
        if (ua > 0 && !warp_wait(afree + sl, (ua - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const uint4 wv = blk ? w1 : w0;
          const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
          uint32_t r[16];
          if (FMT == kFmtFp8) {
            // 64-block blk = tiles 2 blk and 2 blk + 1; k16 sub-block k uses
            // words 2 (k & 1) (P0, P1) and 2 (k & 1) + 1 (P2, P3) of tile
            // 2 blk + (k >> 1); exact e4m3 -> f16, the scale is per tensor
            const uint4 ta = blk ? w2 : w0, tb = blk ? w3 : w1;
            const uint32_t fw[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t wa = fw[2 * k], wb = fw[2 * k + 1];
              r[4 * k + 0] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa));
              r[4 * k + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb));
              r[4 * k + 2] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa >> 16));
              r[4 * k + 3] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb >> 16));
            }
          } else if (FMT == 0) {
            const uint32_t s_lo = prmt(sv0, sv0, 0x1010u);  // (s_g, s_g)
            const uint32_t s_hi = prmt(sv0, sv0, 0x3232u);  // (s_g8, s_g8)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // register order of 16x256b: (row g, col 2t), (row g, col 2t+1),
              // (row g+8, col 2t), (row g+8, col 2t+1) = P0, P2, P1, P3
              r[4 * k + 0] = hmul2_bf16(int4_pair_to_bf16x2(wd[k]), s_lo);
              r[4 * k + 1] = hmul2_bf16(int4_pair_to_bf16x2(wd[k] >> 8), s_lo);
              r[4 * k + 2] = hmul2_bf16(int4_pair_to_bf16x2(wd[k] >> 4), s_hi);
              r[4 * k + 3] = hmul2_bf16(int4_pair_to_bf16x2(wd[k] >> 12), s_hi);
            }
          } else {
            const uint32_t sw2[2] = {blk ? sv2 : sv0, blk ? sv3 : sv1};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t s2 =
                  e4m3x2_to_f16x2(static_cast<uint16_t>(sw2[k >> 1] >> (16 * (k & 1))));
              const uint32_t s_lo = prmt(s2, s2, 0x1010u), s_hi = prmt(s2, s2, 0x3232u);
              r[4 * k + 0] = hmul2_f16(e2m1x2_to_f16x2(wd[k]), s_lo);
              r[4 * k + 1] = hmul2_f16(e2m1x2_to_f16x2(wd[k] >> 16), s_lo);
              r[4 * k + 2] = hmul2_f16(e2m1x2_to_f16x2(wd[k] >> 8), s_hi);
              r[4 * k + 3] = hmul2_f16(e2m1x2_to_f16x2(wd[k] >> 24), s_hi);
            }
          }
          tmem_st_16x256b_x4(a_base + sl * 128 + blk * 32, r);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull + sl);
        if (++sl == kASlots) {
          sl = 0;
          ++ua;
        }
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue of a unit
      if (!warp_wait(dfull, unit_i & 1, abort_flag, p.err)) break;
      tc_fence_after();
      constexpr int kHalf = MPAD / 2;                   // columns this warp reads
      constexpr int kEC = kHalf % 32 == 0 ? 32 : kHalf % 16 == 0 ? 16 : 8;   // per tcgen05.ld
      // weight row of this lane; fused: gate row i in half 0, up row I + i in half 1
      const int i_out = tile * (p.fuse ? 128 : kTcTileRows) + (p.fuse ? 0 : h * 128) + 32 * q + lane;
      const int n = p.fuse ? (h ? p.I : 0) + i_out : i_out;
      const bool n_ok = p.fuse ? i_out < p.I : n < p.N;
      const int m0 = bp * kHalf;                        // local row of the chunk
      const int xrow = chunk * p.rows;
      const int mlim = min(p.rows, p.M - xrow);          // rows of this chunk
      float gmul = 1.f;
      if (FMT != 0) gmul = __ldg(p.g);                   // NVFP4 and FP8: per-tensor scale
      const size_t Npad = (size_t)p.NT * 16;
      if (p.fuse && p.S == 1) {
        // fused, not split: every warp reads gate (half 0) and up (half 1) for
        // its 32 lanes, which hold the same output row i, over a quarter of
        // the columns, and writes BF16(SiLU(gate) * up)
        constexpr int kQ = MPAD / 4;
        constexpr int kEQ = kQ % 32 == 0 ? 32 : kQ % 16 == 0 ? 16 : kQ % 8 == 0 ? 8 : 4;
        const int mq = (2 * bp + h) * kQ;
        const int i_row = tile * 128 + 32 * q + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < kQ; c0 += kEQ) {
          float v[kEQ], u[kEQ];
          tmem_ld_32x32b<kEQ>(tmem + ((uint32_t)(32 * q) << 16) + mq + c0, v);
          tmem_ld_32x32b<kEQ>(tmem + ((uint32_t)(32 * q) << 16) + kDStride + mq + c0, u);
          tmem_wait_ld();
          if (i_row < p.I) {
            const int mb = xrow + mq + c0;
            __nv_bfloat16* hp = p.y + (size_t)mb * p.I + i_row;
#pragma unroll
            for (int c = 0; c < kEQ; ++c, hp += p.I) {
              if (mq + c0 + c < mlim) {
                float gv = v[c], uv = u[c];
                if (FMT != 0) {
                  const float rm = __ldg(p.row_mul + mb + c);
                  gv = gv * rm * gmul;
                  uv = uv * rm * gmul;
                }
                *hp = __float2bfloat16_rn(silu_f32(gv) * uv);
              }
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < kHalf; c0 += kEC) {
          float v[kEC];
          tmem_ld_32x32b<kEC>(tmem + ((uint32_t)(32 * q) << 16) + h * kDStride + m0 + c0, v);
          tmem_wait_ld();
          if (n_ok) {
            const int mb = xrow + m0 + c0;                 // first row of this batch
            if (p.S == 1) {
              __nv_bfloat16* yp = p.y + (size_t)mb * p.N + n;
#pragma unroll
              for (int c = 0; c < kEC; ++c, yp += p.N) {
                if (m0 + c0 + c < mlim) {
                  float val = v[c];
                  if (FMT != 0) val = val * __ldg(p.row_mul + mb + c) * gmul;
                  *yp = __float2bfloat16_rn(val);
                }
              }
            } else {
              float* wp = p.ws + ((size_t)split * p.M + mb) * Npad + n;
#pragma unroll
              for (int c = 0; c < kEC; ++c, wp += Npad)
                if (m0 + c0 + c < mlim) __stcg(wp, v[c]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dfree);
    }
    cpa_wait<0>();  // no copy in flight at exit
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// Per-row power-of-two rescaling of the activations into FP16 (NVFP4 and
// FP8 paths): row_mul[m] = 2^e with max|x[m]| * 2^-e in [2^14, 2^15).  One
// CTA per row, eight BF16 values per 16-byte load; the second pass re-reads
// the row from cache.  K is a multiple of 128, so rows are 16-byte aligned.
// Launched with programmatic dependent launch: the tensor-core kernel may
// start at once, and this kernel reads x (and overwrites the FP16 copy the
// previous call may still be reading) only after the previous kernel on the
// stream has finished.
__global__ void __launch_bounds__(256) prep_x_f16_kernel(const __nv_bfloat16* __restrict__ x,
                                                         __half* __restrict__ xh,
                                                         float* __restrict__ row_mul, int K) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)m * K);
  uint4* out = reinterpret_cast<uint4*>(xh + (size_t)m * K);
  const int n8 = K >> 3;
  float mx = 0.f;
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = __ldg(row + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      mx = fmaxf(mx, fabsf(__uint_as_float(w[j] << 16)));
      mx = fmaxf(mx, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
    }
  }
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    mx = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (threadIdx.x == 0) red[0] = mx;
  }
  __syncthreads();
  mx = red[0];
  int e = 0;
  if (mx > 0.f && isfinite(mx)) e = ilogbf(mx) - 14;
  if (threadIdx.x == 0) row_mul[m] = ldexpf(1.f, e);
  // x * 2^-e is one exact scaling: a single multiply when 2^-e is a normal
  // float, ldexpf otherwise (rows whose largest magnitude is below 2^-112)
  const bool direct = e >= -126 && e <= 126;
  const float sc = direct ? __int_as_float((127 - e) << 23) : 0.f;
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = __ldg(row + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      const __half hl = __float2half_rn(direct ? lo * sc : ldexpf(lo, -e));
      const __half hh = __float2half_rn(direct ? hi * sc : ldexpf(hi, -e));
      o[j] = (uint32_t)__half_as_ushort(hl) | ((uint32_t)__half_as_ushort(hh) << 16);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Split-K reduction: y[m][n] = BF16(sum over splits, in split order, of the
// fp32 partials [S][M][Npad]), times the NVFP4 row multiplier and global
// scale.  Four columns per thread; launched behind the main kernel with
// programmatic dependent launch, so it waits for the partials on the device.
// Sum over splits, in split order, of four consecutive partials at `src`.
__device__ __forceinline__ void sum_splits4(const float* src, size_t sstride, int S, float* a) {
  a[0] = a[1] = a[2] = a[3] = 0.f;
  int sp = 0;
  for (; sp + 4 <= S; sp += 4) {                 // four splits' loads in flight, added in order
    float4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = __ldcg(reinterpret_cast<const float4*>(src + (sp + j) * sstride));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a[0] += v[j].x;
      a[1] += v[j].y;
      a[2] += v[j].z;
      a[3] += v[j].w;
    }
  }
  for (; sp < S; ++sp) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(src + sp * sstride));
    a[0] += v.x;
    a[1] += v.y;
    a[2] += v.z;
    a[3] += v.w;
  }
}

// Fused gate/up: `cols` = I output columns, gate partials at n, up at I + n,
// y[m][n] = BF16(SiLU(gate) * up).
template <int FMT, bool FUSE>
__global__ void __launch_bounds__(256)
    tc_splitk_reduce(const float* __restrict__ ws, int S, int M, int cols, int Npad,
                     const float* __restrict__ row_mul, const float* __restrict__ g,
                     __nv_bfloat16* __restrict__ y) {
  // a following GEMM may start streaming its weights now (it waits for this
  // grid before it touches anything this grid reads or writes)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int m = blockIdx.y;
  const int n0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (n0 >= cols) return;
  const size_t sstride = (size_t)M * Npad;
  float a[4], u[4];
  sum_splits4(ws + (size_t)m * Npad + n0, sstride, S, a);
  if (FUSE) sum_splits4(ws + (size_t)m * Npad + cols + n0, sstride, S, u);
  float rm = 1.f, gm = 1.f;
  if (FMT != 0) {
    rm = __ldg(row_mul + m);
    gm = __ldg(g);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (n0 + j < cols) {
      float val = a[j];
      if (FMT != 0) val = val * rm * gm;
      if (FUSE) {
        float uv = u[j];
        if (FMT != 0) uv = uv * rm * gm;
        val = silu_f32(val) * uv;
      }
      y[(size_t)m * cols + n0 + j] = __float2bfloat16_rn(val);
    }
  }
}

// Diagnostics: two warps wait, through the same bounded waits the kernel
// above uses, on an mbarrier that nothing arrives at.  The first to exhaust
// its bound records the timeout in the device error word and raises the
// CTA's abort flag; the other sees the flag and gives up without waiting out
// its own bound.  out[w] = 1 if warp w's wait returned false.
__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(unsigned* err, int* out) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = warp_wait(&bar, 0, &abort_flag, err);
  if ((threadIdx.x & 31) == 0) out[threadIdx.x >> 5] = ok ? 0 : 1;
}

// ------------------------------------------------------------------ host side

bool make_xmap(CUtensorMap* map, const void* x, int M, int K, int mpad, bool f16) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)mpad};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


template <int FMT, int MPAD>
cudaError_t launch_t(const TcPlan& pl, const GemmArgs& a, const void* xsrc, const float* row_mul,
                     cudaStream_t st) {
  CUtensorMap map;
  if (!make_xmap(&map, xsrc, a.M, a.K, MPAD, FMT != 0)) return cudaErrorInvalidValue;
  TcParams p;
  p.w = static_cast<const uint8_t*>(a.w);
  p.s = static_cast<const uint8_t*>(a.s);
  p.g = a.g;
  p.row_mul = row_mul;
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.ws = a.ws;
  p.err = a.err;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.KB = a.K / 64;
  p.NT = (a.N + 15) / 16;
  p.fuse = a.fuse;
  p.I = a.N / 2;
  p.tiles = a.fuse ? (p.I + 127) / 128 : (a.N + kTcTileRows - 1) / kTcTileRows;
  p.S = pl.S;
  p.gps = pl.kbs / 2;
  p.chunks = pl.chunks;
  p.rows = pl.rows;
  p.units = p.tiles * pl.chunks * pl.S;
  // the dynamic shared memory limit, raised once per device and variant (an
  // atomic flag: host threads may race here; the attribute call is idempotent)
  static std::atomic<int> smem_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem_set[dev].load(std::memory_order_acquire) < pl.smem) {
    cudaError_t e =
        cudaFuncSetAttribute(tc_kernel<FMT, MPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return e;
    int cur = smem_set[dev].load(std::memory_order_relaxed);
    while (cur < pl.smem && !smem_set[dev].compare_exchange_weak(cur, pl.smem)) {
    }
  }
  // Programmatic dependent launch: on each SM freed by the previous kernel
  // (for NVFP4 and FP8, the FP16 rescale kernel, itself launched the same
  // way) the CTA starts (tensor memory, barriers, an L2 prefetch of its first
  // weights) before that kernel has finished; every read of an operand and
  // every write waits for it (griddepcontrol.wait).  Measured 3-8 % faster
  // back to back for int4.
  cudaLaunchConfig_t kcfg = {};
  kcfg.gridDim = dim3((unsigned)pl.grid, 1, 1);
  kcfg.blockDim = dim3(kTcThreads, 1, 1);
  kcfg.dynamicSmemBytes = (size_t)pl.smem;
  kcfg.stream = st;
  cudaLaunchAttribute kattr[1];
  kattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  kattr[0].val.programmaticStreamSerializationAllowed = 1;
  kcfg.attrs = kattr;
  kcfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&kcfg, tc_kernel<FMT, MPAD>, map, p);
  if (e != cudaSuccess || pl.S == 1) return e;

  const int cols = a.fuse ? a.N / 2 : a.N;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((cols + 1023) / 1024), (unsigned)a.M, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* ws = a.ws;
  __nv_bfloat16* y = static_cast<__nv_bfloat16*>(a.y);
  if (a.fuse)
    return cudaLaunchKernelEx(&cfg, tc_splitk_reduce<FMT, true>, ws, pl.S, a.M, cols, p.NT * 16,
                              row_mul, a.g, y);
  return cudaLaunchKernelEx(&cfg, tc_splitk_reduce<FMT, false>, ws, pl.S, a.M, cols, p.NT * 16,
                            row_mul, a.g, y);
}

template <int FMT>
cudaError_t launch_fmt(const TcPlan& pl, const GemmArgs& a, const void* xsrc, const float* rm,
                       cudaStream_t st) {
  switch (pl.mpad) {
    case 16: return launch_t<FMT, 16>(pl, a, xsrc, rm, st);
    case 32: return launch_t<FMT, 32>(pl, a, xsrc, rm, st);
    case 48: return launch_t<FMT, 48>(pl, a, xsrc, rm, st);
    case 64: return launch_t<FMT, 64>(pl, a, xsrc, rm, st);
    case 80: return launch_t<FMT, 80>(pl, a, xsrc, rm, st);
    case 96: return launch_t<FMT, 96>(pl, a, xsrc, rm, st);
    case 112: return launch_t<FMT, 112>(pl, a, xsrc, rm, st);
    default: return launch_t<FMT, 128>(pl, a, xsrc, rm, st);
  }
}

template <int MPAD>
int tc_smem(int fmt) {
  return fmt == 0 ? TcShape<0, MPAD>::kSmem
         : fmt == 1 ? TcShape<1, MPAD>::kSmem : TcShape<kFmtFp8, MPAD>::kSmem;
}

}  // namespace

// Splits K so that the units (256-row tiles x row chunks x K splits, whole
// 128-groups each) fill the SMs.  Estimated time in microseconds, from
// per-group and per-unit timings of the kernel on B200 (clock64 timelines):
// the busiest CTA's waves x (its groups x t_group + t_unit), t_unit being the
// epilogue and pipeline refill of a unit, plus, with split K, the reduction
// launch and its traffic (the partials written and read once more).
TcPlan plan_tc(int fmt, int M, int N, int K, int num_sms, int fuse) {
  TcPlan pl;
  pl.chunks = (M + kTcMaxRows - 1) / kTcMaxRows;
  pl.rows = (M + pl.chunks - 1) / pl.chunks;
  pl.mpad = (pl.rows + 15) / 16 * 16;
  const int tiles = fuse ? (N / 2 + 127) / 128 : (N + kTcTileRows - 1) / kTcTileRows;
  const int groups = K / 128;
  const double t_group = 0.75 + 0.0017 * pl.mpad;   // us per 128-group of a 256-row tile
  const double t_unit = 0.5 + 0.035 * pl.mpad;      // us per unit: epilogue, refill
  const double part_mb = (double)M * ((N + 15) / 16 * 16) * 4 / 1e6;   // one split's partials
  double best = 1e300;
  int best_s = 1;
  for (int S = 1; S <= 16 && S <= groups; ++S) {
    const int gps = (groups + S - 1) / S;
    if ((S - 1) * gps >= groups) continue;
    const int units = tiles * pl.chunks * S;
    const int waves = (units + num_sms - 1) / num_sms;
    const double cost = waves * (gps * t_group + t_unit) + (S > 1 ? 2.0 + S * part_mb / 3.0 : 0.0);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = S;
    }
  }
  pl.S = best_s;
  pl.kbs = 2 * ((groups + pl.S - 1) / pl.S);
  pl.units = tiles * pl.chunks * pl.S;
  pl.grid = pl.units < num_sms ? pl.units : num_sms;
  int smem = 0;
  switch (pl.mpad) {
    case 16: smem = tc_smem<16>(fmt); break;
    case 32: smem = tc_smem<32>(fmt); break;
    case 48: smem = tc_smem<48>(fmt); break;
    case 64: smem = tc_smem<64>(fmt); break;
    case 80: smem = tc_smem<80>(fmt); break;
    case 96: smem = tc_smem<96>(fmt); break;
    case 112: smem = tc_smem<112>(fmt); break;
    default: smem = tc_smem<128>(fmt); break;
  }
  pl.smem = smem;
  return pl;
}

size_t tc_workspace_floats(const TcPlan& p, int M, int N) {
  return p.S > 1 ? static_cast<size_t>(p.S) * M * ((N + 15) / 16 * 16) : 0;
}

size_t tc_counters(const TcPlan& p, int N) {
  (void)p;
  (void)N;
  return 0;   // the split-K reduction is a separate kernel: no arrival counters
}

size_t tc_x_f16_bytes(int fmt, int M, int K) {
  return fmt != 0 ? (size_t)M * K * 2 + (size_t)M * sizeof(float) : 0;
}

// NVFP4 and FP8 first rescale all M rows into FP16 (one launch); then one launch of
// the tensor-core kernel covers every chunk of rows (plus, when K is split,
// one reduction launch).
cudaError_t launch_tc(const TcPlan& pl, const GemmArgs& a, void* xf16_scratch, cudaStream_t st) {
  if (a.fmt == 0) return launch_fmt<0>(pl, a, a.x, nullptr, st);
  __half* xh = static_cast<__half*>(xf16_scratch);
  float* rm = reinterpret_cast<float*>(static_cast<uint8_t*>(xf16_scratch) + (size_t)a.M * a.K * 2);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.M, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prep_x_f16_kernel, static_cast<const __nv_bfloat16*>(a.x),
                                     xh, rm, a.K);
  if (e != cudaSuccess) return e;
  return a.fmt == 1 ? launch_fmt<1>(pl, a, xh, rm, st) : launch_fmt<kFmtFp8>(pl, a, xh, rm, st);
}

cudaError_t launch_wait_timeout_selftest(unsigned* err, int* out, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 64, 0, st>>>(err, out);
  return cudaGetLastError();
}

}  // namespace w4
