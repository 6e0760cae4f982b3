// Split-K weight-streaming GEMV for decode row counts (M <= 16) on sm_100a.
//
// Why this shape: at small M the matmul moves ~0.5 byte of packed weight per
// 2*M flops, so the time is the time to stream the weights from HBM once (the
// bandwidth argument of the blog post "One Config Line Made My 27B Model 2.7x
// Faster", section "Gotcha #2").  The kernel's job is to keep enough bytes in
// flight and to spend as few instructions per weight as possible turning
// nibbles into multiply operands: at 7+ TB/s a B200 SM has about two
// lane-instructions per weight.
//
// Structure (one CTA of 16 warps per SM):
//  * A CTA owns one K-slice and a contiguous range of 16-row bands.  Its
//    warps form a (Wn x Wk) grid: Wn bands in flight at a time, each band's
//    slice cut into Wk group-aligned pieces, one per warp.  The Wk partial
//    sums of a band are added in piece order through shared memory
//    (deterministic).
//  * Each warp streams its pieces, one 128-group (two 512-byte tiles and
//    their scales) at a time, through its own ring of shared-memory stages
//    filled by cp.async: every lane copies, and later reads back, exactly its
//    own 16 bytes of each tile (a warp's copies cover the whole tile), so no
//    barrier guards the ring; only the lane's own cp.async groups are waited
//    for.  The ring holds up to eight groups per warp (up to 144 KB per SM
//    in flight) without spending registers, and runs on from one band's
//    piece into the next.  Under programmatic dependent launch the CTA starts
//    before the previous kernel on the stream has finished but then only
//    prefetches its first weights and the activations into L2: any operand
//    may have been written by that kernel, so every read into the SM comes
//    after griddepcontrol.wait.
//  * The CTA copies its slice of the activations into shared memory as FP16,
//    each row rescaled by a power of two so that its largest magnitude lies in
//    [2^14, 2^15) (exact for every BF16 value in FP16's normal range), k
//    reordered inside every 16-block to match the packed operand fragments.
//  * Per 32-bit word (8 weights) a lane builds the A fragment of one
//    mma.sync m16n8k16 (16 output columns x 16 k) with exact FP16 arithmetic:
//    int4: 1 shift, 4 LOP3 that drop each nibble into the mantissa of FP16
//    1024.0, then 4 subtractions / fused multiply-adds that leave q; NVFP4:
//    4 hardware e2m1 -> f16 conversions; FP8-E4M3 (two words per 16 k): 4
//    hardware e4m3 -> f16 conversions.  The activations are the n8 side:
//    one MMA serves 8 rows.  Group scales multiply the fp32 MMA results
//    (int4: once per 128-group, NVFP4: once per 16-group); the per-tensor
//    scale of NVFP4 and FP8 is applied in the epilogue.
//  * Split-K partials across CTAs go to a fp32 workspace; the last CTA to
//    finish a band (arrival counter) adds them in split order.
//  * Fused gate/up layer (FUSE): each ring stage also holds the up band's
//    group, a second accumulator set takes it, and the epilogue writes
//    SiLU(gate) * up.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace w4 {

namespace {

constexpr int kRowWords = 64;                                // per-row words (M <= 64)
constexpr int kRowAuxOff = kRowWords * 4;
constexpr int kBarOff = 2 * kRowWords * 4;                   // mbarrier of the activation copy
constexpr int kRedOff = kBarOff + 128;                       // per-lane partial sums
constexpr int kMaxSmem = 232448;                             // 227 KB opt-in
constexpr int kMaxDepth = 8;                                 // ring stages per warp
constexpr int kGroupBytes = 2 * kTileBytes;                  // packed 4-bit weights of one band-group

// Packed weights of one band's 128-group: two 512-byte tiles at 4 bits, four at 8.
__host__ __device__ constexpr int group_bytes(int fmt) { return fmt == kFmtFp8 ? 4 * kTileBytes : kGroupBytes; }

// Shared-memory bytes of one ring stage: the group's two tiles, then the
// scales each lane needs (int4: 4 bytes, NVFP4: 2 x 8 bytes per lane).
__host__ __device__ constexpr int stage_bytes(int fmt) {
  return fmt == kFmtFp8 ? group_bytes(fmt) : kGroupBytes + (fmt == 0 ? 128 : 512);
}

// Warps per CTA: a power of two (the warp grid is split with shifts).  16
// warps leave 128 registers a thread; with 64 (32 warps) the compiler
// rematerialises the conversion constants in the loop, and the ring, not the
// warp count, keeps the bytes in flight (measured: 16 warps are ~20% faster
// at M = 1).
template <int FMT, int MT, bool FUSE = false>
struct Cfg {
  static constexpr int kWarps = 16;
  static constexpr int kRedBytes = kWarps * 32 * 4 * MT * 4 * (FUSE ? 2 : 1);  // per-lane partial sums
  static constexpr int kHeader = (kRedOff + kRedBytes + 127) / 128 * 128;
};

struct Params {
  const __nv_bfloat16* x;
  const uint8_t* w;
  const uint8_t* s;
  const float* g;
  __nv_bfloat16* y;
  float* ws;
  unsigned* counters;
  unsigned* err;
  int M, N, K, NT, S, kslice, row_stride;          // row_stride in bytes
  int stage_log2;                                  // log2 of the staging threads per row
  int bq, br;                                      // bands per CTA: bq, plus one for the first br
  int wn, wn_log2, wk_log2;                        // warp grid: wn bands x 2^wk_log2 pieces
  int ngp;                                         // groups per piece, padded to the ring depth
  // fused gate/up layer: bands index the I gate rows; the up band of gate
  // band b lies up_w (weights) and up_s (scales) bytes further; y is [M][I]
  int I;
  size_t up_w, up_s;
};


// Programmatic dependent launch: let the next kernel on the stream start its
// prologue, and wait for the previous one before touching data it may write.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ cp.async

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
// Wait until at most N of this thread's cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cpa_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ activations

// Element kin of a 64-block sits at this element offset of the block's image
// in shared memory: lane t reads 16 contiguous elements k = 16 j + 4 t + e.
__device__ __forceinline__ int perm64(int kin) {
  const int j = kin >> 4, t = (kin >> 2) & 3, e = kin & 3;
  return t * 16 + j * 4 + e;
}

// Lane-wise maximum of two pairs of unsigned 16-bit integers.
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 1-D bulk copy global -> shared completing on an mbarrier (no multicast):
// both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Hint: bring a byte range into L2 (no data is returned to the SM, so it may
// run before the previous kernel on the stream has finished writing it).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// The CTA's slice of the activations as the FP16 image (see the file
// comment).  Warp 0 has bulk-copied each row's raw BF16 slice into that row
// of the image (completing on xbar); this waits for it, takes every row's
// largest magnitude, and rewrites each 64-block in place as FP16 scaled by
// the row's power of two, k permuted.  Every row has 2^stage_log2 threads (a
// power of two, at least a warp; rows past M have idle threads), so a warp's
// 32 lanes always hold the 8 chunks (16 bytes each) of 4 whole blocks of one
// row and the in-place rewrite of a block needs only the warp itself.  All
// 16 warps run this at once, so its cost is its instruction count: no
// divisions, 32-bit offsets.  row_aux must be zero and visible on entry.
// Ends with a barrier after which the image and row_mul are valid.  Returns
// false if the copy did not complete (bounded wait).
__device__ bool stage_activations(const Params& p, int k_len, uint8_t* xs, float* row_mul,
                                  unsigned* row_aux, uint64_t* xbar) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // warp 0 waits for the copy (converged again before the barrier), the
  // others at the barrier
  bool ok_w = true;
  if (warp == 0) {
    ok_w = mbar_wait(xbar, 0, p.err);
    ok_w = __all_sync(0xffffffffu, ok_w);
  }
  const bool ok = __syncthreads_and(ok_w) != 0;
  const int tpr = 1 << p.stage_log2;
  const int m = threadIdx.x >> p.stage_log2;
  const int c_first = (threadIdx.x & (tpr - 1)) - lane;      // this warp's first chunk of the row
  const int cpr = k_len >> 3;                                 // 16-byte chunks per row
  uint8_t* row = xs + m * p.row_stride;
  if (m < p.M) {
    // magnitudes compared as integers (BF16 bits with the sign cleared order
    // like the values), two per instruction
    uint32_t mx = 0u;
    for (int c = c_first + lane; c < cpr; c += tpr) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + c * 16);
      mx = vmax_u16x2(mx, vmax_u16x2(vmax_u16x2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                     vmax_u16x2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
    }
    const unsigned r = __reduce_max_sync(0xffffffffu, max(mx & 0xFFFFu, mx >> 16));
    if (lane == 0) atomicMax(row_aux + m, r << 16);           // fp32 bits of the BF16 value
  }
  __syncthreads();
  if (m < p.M) {
    const float rmax = __uint_as_float(row_aux[m]);
    const bool scaled = rmax > 0.f && isfinite(rmax);
    // max * 2^sh in [2^14, 2^15); |sh| <= 126 keeps 2^sh and 2^-sh normal floats
    // (rows whose largest magnitude is below 2^-112 keep fewer FP16 bits)
    const int sh = scaled ? min(126, 14 - ilogbf(rmax)) : 0;
    const float mul = __int_as_float((127 + sh) << 23);       // 2^sh, exact
    if (c_first + lane == 0) row_mul[m] = __int_as_float((127 - sh) << 23);   // 2^-sh
    for (int c0 = c_first; c0 < cpr; c0 += tpr) {
      const int c = c0 + lane;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (c < cpr) v = *reinterpret_cast<const uint4*>(row + c * 16);
      __syncwarp();                                 // the 4 blocks are read before any is rewritten
      if (c < cpr) {
        uint32_t out[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = __uint_as_float(out[e] << 16) * mul;
          const float hi = __uint_as_float(out[e] & 0xFFFF0000u) * mul;
          __half2 h = __floats2half2_rn(lo, hi);
          out[e] = *reinterpret_cast<uint32_t*>(&h);
        }
        uint8_t* blk = row + (c >> 3) * 128;
        const int in = (c & 7) * 8;
        // the first half of a chunk lands in banks 0-7 / 16-23 of its block,
        // the second in 8-15 / 24-31: odd blocks store them in the other
        // order, so each half-warp's stores cover all 32 banks once
        const bool odd = (c >> 3) & 1;
        const uint2 first = odd ? make_uint2(out[2], out[3]) : make_uint2(out[0], out[1]);
        const uint2 second = odd ? make_uint2(out[0], out[1]) : make_uint2(out[2], out[3]);
        *reinterpret_cast<uint2*>(blk + perm64(in + (odd ? 4 : 0)) * 2) = first;
        *reinterpret_cast<uint2*>(blk + perm64(in + (odd ? 0 : 4)) * 2) = second;
      }
      __syncwarp();
    }
  }
  __syncthreads();
  return ok;
}

// c = A . B (fresh accumulator), fp32
__device__ __forceinline__ void mma_f16_first(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// The words a lane needs for one 128-group of one band.
struct GroupWords {
  uint4 w0, w1;   // the two 64-blocks
  uint2 s0, s1;   // int4: s0.x = scales of rows g, g+8; NVFP4: per-block E4M3 scales
};

// One 128-group of one band, int4.  xg[mt]: this lane's activation fragment
// of the group's first 64-block for 8-row tile mt (the second block follows
// 128 bytes later).
template <int MT>
__device__ __forceinline__ void group_int4(const GroupWords& gw, const uint8_t* const* xg,
                                           float (*acc)[4]) {
  const float s_lo = __uint_as_float(gw.s0.x << 16);          // row g
  const float s_hi = __uint_as_float(gw.s0.x & 0xFFFF0000u);  // row g + 8
  float c[2][MT][4];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint4 wv = half ? gw.w1 : gw.w0;
    const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t a[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // FP16 holds two nibbles per 16-bit half in its mantissa: one shift per word
      const uint32_t hi = wd[j] >> 8;
      a[j][0] = int4_lo_pair_to_f16x2(wd[j]);
      a[j][1] = int4_hi_pair_to_f16x2(wd[j]);
      a[j][2] = int4_lo_pair_to_f16x2(hi);
      a[j][3] = int4_hi_pair_to_f16x2(hi);
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const uint4* xb = reinterpret_cast<const uint4*>(xg[mt] + half * 128);
      const uint4 v0 = xb[0], v1 = xb[1];
      const uint32_t bx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      mma_f16_first(c[half][mt], a[0], bx[0], bx[1]);
#pragma unroll
      for (int j = 1; j < 4; ++j) mma_f16_16816(c[half][mt], a[j], bx[2 * j], bx[2 * j + 1]);
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    acc[mt][0] = fmaf(s_lo, c[0][mt][0] + c[1][mt][0], acc[mt][0]);
    acc[mt][1] = fmaf(s_lo, c[0][mt][1] + c[1][mt][1], acc[mt][1]);
    acc[mt][2] = fmaf(s_hi, c[0][mt][2] + c[1][mt][2], acc[mt][2]);
    acc[mt][3] = fmaf(s_hi, c[0][mt][3] + c[1][mt][3], acc[mt][3]);
  }
}

// One 64-block of one band, NVFP4 (a scale per 16-group, i.e. per MMA).  wv:
// this lane's words of the tile; sv: E4M3 scales of rows g and g+8, 4 groups.
template <int MT>
__device__ __forceinline__ void block_nvfp4(uint4 wv, uint2 sv, const uint8_t* const* xb0,
                                            float (*acc)[4]) {
  const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
  uint32_t a[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    a[j][0] = e2m1x2_to_f16x2(wd[j]);
    a[j][1] = e2m1x2_to_f16x2(wd[j] >> 8);
    a[j][2] = e2m1x2_to_f16x2(wd[j] >> 16);
    a[j][3] = e2m1x2_to_f16x2(wd[j] >> 24);
  }
  const uint32_t sw2[2] = {sv.x, sv.y};
  float2 sf[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint16_t>(sw2[j >> 1] >> (16 * (j & 1))));
    sf[j] = __half22float2(*reinterpret_cast<const __half2*>(&s2));
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const uint4* xb = reinterpret_cast<const uint4*>(xb0[mt]);
    const uint4 v0 = xb[0], v1 = xb[1];
    const uint32_t bx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float c[4];
      mma_f16_first(c, a[j], bx[2 * j], bx[2 * j + 1]);
      acc[mt][0] = fmaf(sf[j].x, c[0], acc[mt][0]);
      acc[mt][1] = fmaf(sf[j].x, c[1], acc[mt][1]);
      acc[mt][2] = fmaf(sf[j].y, c[2], acc[mt][2]);
      acc[mt][3] = fmaf(sf[j].y, c[3], acc[mt][3]);
    }
  }
}

// One 128-group of one band, FP8-E4M3 (per-tensor scale, applied in the
// epilogue): st is this lane's 16 bytes of the group's first tile; the four
// tiles are 512 bytes apart, two per 64-block, two k16 sub-blocks per tile.
template <int MT>
__device__ __forceinline__ void group_fp8(const uint8_t* st, const uint8_t* const* xg,
                                          float (*acc)[4]) {
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    const uint4 t0 = *reinterpret_cast<const uint4*>(st + (2 * blk) * kTileBytes);
    const uint4 t1 = *reinterpret_cast<const uint4*>(st + (2 * blk + 1) * kTileBytes);
    const uint32_t wd[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
    uint32_t a[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {     // k16 sub-block j of the 64-block: words 2j (P0, P1), 2j+1 (P2, P3)
      a[j][0] = e4m3x2_to_f16x2(static_cast<uint16_t>(wd[2 * j]));
      a[j][1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wd[2 * j] >> 16));
      a[j][2] = e4m3x2_to_f16x2(static_cast<uint16_t>(wd[2 * j + 1]));
      a[j][3] = e4m3x2_to_f16x2(static_cast<uint16_t>(wd[2 * j + 1] >> 16));
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const uint4* xb = reinterpret_cast<const uint4*>(xg[mt] + blk * 128);
      const uint4 v0 = xb[0], v1 = xb[1];
      const uint32_t bx[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) mma_f16_16816(acc[mt], a[j], bx[2 * j], bx[2 * j + 1]);
    }
  }
}

template <int FMT, int MT, bool FUSE>
__device__ __forceinline__ void band_epilogue(const Params& p, int band, int split, int lane,
                                              const float* row_mul, const float (*vals)[4],
                                              const float (*vals_u)[4]) {
  const int g = lane >> 2, t = lane & 3;
  const float gmul = FMT != 0 ? __ldg(p.g) : 1.f;   // NVFP4 and FP8: per-tensor scale
  const int n0 = band * 16 + g;
  const int cols = FUSE ? p.I : p.N;             // output columns (row stride of y)
  if (p.S == 1) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = mt * 8 + 2 * t + (i & 1);
        const int n = n0 + 8 * (i >> 1);
        if (m < p.M && n < cols) {
          float v = vals[mt][i] * row_mul[m] * gmul;
          if (FUSE) v = silu_f32(v) * (vals_u[mt][i] * row_mul[m] * gmul);
          p.y[(size_t)m * cols + n] = __float2bfloat16_rn(v);
        }
      }
    return;
  }
  // partials [S][M][Npad]: fused, gate row n and up row I + n
  const size_t Npad = FUSE ? (size_t)2 * p.I : (size_t)p.NT * 16;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = mt * 8 + 2 * t + (i & 1);
      const int n = n0 + 8 * (i >> 1);
      if (m < p.M) {
        float* dst = p.ws + ((size_t)split * p.M + m) * Npad + n;
        __stcg(dst, vals[mt][i] * row_mul[m]);
        if (FUSE) __stcg(dst + p.I, vals_u[mt][i] * row_mul[m]);
      }
    }
  __threadfence();
  __syncwarp();
  unsigned prev = 0;
  if (lane == 0) prev = atomicAdd(p.counters + band, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != static_cast<unsigned>(p.S - 1)) return;
  __threadfence();
  // sum the splits in split order; the loads of kB splits are issued
  // together (one round trip per batch instead of one per split)
  constexpr int kV = MT * 4 * (FUSE ? 2 : 1);          // values of this lane
  constexpr int kB = 32 / kV;                          // 32 loads in flight per lane
  float sum[kV];
#pragma unroll
  for (int j = 0; j < kV; ++j) sum[j] = 0.f;
  const size_t sstride = (size_t)p.M * Npad;
  for (int sp0 = 0; sp0 < p.S; sp0 += kB) {
    float part[kB][kV];
#pragma unroll
    for (int b = 0; b < kB; ++b)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = mt * 8 + 2 * t + (i & 1);
          const int n = n0 + 8 * (i >> 1);
          const bool ld = sp0 + b < p.S && m < p.M && n < cols;
          const float* src = p.ws + (size_t)(sp0 + b) * sstride + (size_t)m * Npad + n;
          part[b][mt * 4 + i] = ld ? __ldcg(src) : 0.f;
          if (FUSE) part[b][MT * 4 + mt * 4 + i] = ld ? __ldcg(src + p.I) : 0.f;
        }
#pragma unroll
    for (int b = 0; b < kB; ++b)
#pragma unroll
      for (int j = 0; j < kV; ++j) sum[j] += part[b][j];
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = mt * 8 + 2 * t + (i & 1);
      const int n = n0 + 8 * (i >> 1);
      if (m < p.M && n < cols) {
        float v = sum[mt * 4 + i] * gmul;
        if (FUSE) v = silu_f32(v) * (sum[MT * 4 + mt * 4 + i] * gmul);
        p.y[(size_t)m * cols + n] = __float2bfloat16_rn(v);
      }
    }
  if (lane == 0) p.counters[band] = 0u;
}


template <int FMT, int MT, int D, bool FUSE>
__global__ void __launch_bounds__(Cfg<FMT, MT, FUSE>::kWarps * 32, 1) gemv_kernel(const Params p) {
  using C = Cfg<FMT, MT, FUSE>;
  constexpr int kSB1 = stage_bytes(FMT);       // one band's group
  constexpr int kSB = kSB1 * (FUSE ? 2 : 1);   // fused: the gate band's group, then the up band's
  constexpr int kSStep = FMT == 0 ? 32 : FMT == 1 ? 128 : 0;  // scale bytes of a band per 128-group
  constexpr int kGB = group_bytes(FMT);         // weight bytes of a band per 128-group
  constexpr int kTPG = kGB / kTileBytes;        // tiles per group
  extern __shared__ __align__(128) uint8_t smem[];
  float* row_mul = reinterpret_cast<float*>(smem);
  unsigned* row_aux = reinterpret_cast<unsigned*>(smem + kRowAuxOff);
  float* red = reinterpret_cast<float*>(smem + kRedOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* ring = smem + C::kHeader + warp * D * kSB;       // this warp's stages
  uint8_t* xs = smem + C::kHeader + C::kWarps * D * kSB;          // activation image
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + kBarOff);
  if (threadIdx.x < kRowWords) row_aux[threadIdx.x] = 0u;
  if (threadIdx.x == 0) {
    mbar_init(xbar, 1);
    fence_mbar_init();
  }
  pdl_launch_dependents();

  // work of this CTA and warp (no divisions: the host passes quotients and
  // powers of two)
  const int split = blockIdx.y;
  const int k_lo = split * p.kslice;
  const int bx = blockIdx.x;
  const int band_lo = bx * p.bq + min(bx, p.br);
  const int nbands = p.bq + (bx < p.br ? 1 : 0);
  const int wi = warp & (p.wn - 1), wj = warp >> p.wn_log2;
  const int groups = min(p.K - k_lo, p.kslice) >> 7;
  const int g_lo = (wj * groups) >> p.wk_log2, g_hi = ((wj + 1) * groups) >> p.wk_log2;
  const int ng = g_hi - g_lo;                  // real 128-groups in this warp's piece
  const int ngp = p.ngp;                       // padded piece length, a multiple of D
  const int rounds = (nbands + p.wn - 1) >> p.wn_log2;
  const int my_rounds = wi < nbands ? ((nbands - wi - 1) >> p.wn_log2) + 1 : 0;
  const int KB = p.K >> 6;
  const int gk0 = (k_lo >> 7) + g_lo;          // first global 128-group of the piece
  const uint64_t pol = policy_evict_first();

  // Copies run one block of D groups ahead of the reads: the groups of block
  // b + 1 refill the slots of block b as those are read.  A block never spans
  // two bands (pieces are padded to whole blocks), so its groups sit at fixed
  // offsets from one pointer; padding groups copy nothing.
  const int b0 = min(band_lo + wi, p.NT - 1);
  const size_t tpb = (size_t)KB * (kTPG / 2);  // tiles per band
  const uint8_t* cw = p.w + ((size_t)b0 * tpb + kTPG * gk0) * kTileBytes + lane * 16;
  const uint8_t* cs = FMT == 0   ? p.s + ((size_t)b0 * (p.K >> 7) + gk0) * 32 + g * 4
                      : FMT == 1 ? p.s + ((size_t)b0 * KB + 2 * gk0) * 64 + g * 8
                                 : p.s;   // FP8: no packed scales
  // from the last block of a piece to the first block of the next band's piece
  const int wjump = p.wn * (int)tpb * kTileBytes - (ngp - D) * kGB;
  const int sjump = FMT == 0   ? p.wn * (p.K >> 7) * 32 - (ngp - D) * 32
                    : FMT == 1 ? p.wn * KB * 64 - (ngp - D) * 128
                               : 0;
  const int nbp = ngp / D;                     // blocks per piece
  int c_blocks = my_rounds * nbp;              // blocks still to copy
  int c_bb = 0;                                // block index of the cursor within its piece
  const uint32_t ring_s = smem_u32(ring) + lane * 16;
  auto copy_item = [&](int k) {                // group k of the cursor block -> slot k
    if (c_blocks > 0 && c_bb * D + k < ng) {
      const uint32_t d = ring_s + k * kSB;
#pragma unroll
      for (int i = 0; i < kTPG; ++i) cpa16(d + i * kTileBytes, cw + k * kGB + i * kTileBytes, pol);
      if (FMT == 0) {
        cpa4(d + kGroupBytes - lane * 12, cs + k * kSStep);   // scale slot: lane * 4
      } else if (FMT == 1) {
        cpa8(d + kGroupBytes, cs + k * kSStep);
        cpa8(d + kGroupBytes + 8, cs + k * kSStep + 64);
      }
      if (FUSE) {
        const uint8_t* uw = cw + p.up_w + k * kGB;
        const uint8_t* us = cs + p.up_s + k * kSStep;
#pragma unroll
        for (int i = 0; i < kTPG; ++i) cpa16(d + kSB1 + i * kTileBytes, uw + i * kTileBytes, pol);
        if (FMT == 0) {
          cpa4(d + kSB1 + kGroupBytes - lane * 12, us);
        } else if (FMT == 1) {
          cpa8(d + kSB1 + kGroupBytes, us);
          cpa8(d + kSB1 + kGroupBytes + 8, us + 64);
        }
      }
    }
    cpa_commit();
  };
  auto next_block = [&]() {
    if (c_blocks > 0) {
      --c_blocks;
      if (++c_bb == nbp) {
        c_bb = 0;
        cw += wjump;
        cs += sjump;
      } else {
        cw += D * kGB;
        cs += D * kSStep;
      }
    }
  };

  // Before the previous kernel on the stream has finished, only hints: the
  // activation slice and this warp's first block of weights are prefetched
  // into L2.  Any operand may have been written by that kernel (a packer, a
  // previous layer), so nothing is read into the SM before the wait.
  const uint32_t x_bytes = (uint32_t)groups * 256;   // one row's slice, BF16
  if (threadIdx.x < p.M) prefetch_l2(p.x + (size_t)threadIdx.x * p.K + k_lo, x_bytes);
  if (lane == 0 && c_blocks > 0 && ng > 0) {
    const uint32_t n0 = (uint32_t)min(D, ng);        // the block's groups, contiguous from cw
    prefetch_l2(cw, n0 * kGB);
    if (FMT != kFmtFp8) prefetch_l2(cs, n0 * kSStep);
    if (FUSE) {
      prefetch_l2(cw + p.up_w, n0 * kGB);
      if (FMT != kFmtFp8) prefetch_l2(cs + p.up_s, n0 * kSStep);
    }
  }

  pdl_wait();          // the operands may come from the previous kernel
  // the activation copy goes out first (warp 0 initialised its barrier), then
  // the first block of the weight ring
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(xbar, x_bytes * p.M);
    __syncwarp();
    if (lane < p.M)
      bulk_g2s(smem_u32(xs + lane * p.row_stride), p.x + (size_t)lane * p.K + k_lo, x_bytes,
               smem_u32(xbar));
  }
#pragma unroll
  for (int k = 0; k < D; ++k) copy_item(k);
  __syncthreads();     // row_aux zeroed
  const bool x_ok = stage_activations(p, groups * 128, xs, row_mul, row_aux, xbar);
  next_block();

  // activation rows of this lane (row m = 8 mt + g); rows past M alias row 0:
  // their MMA columns are computed but never stored
  const uint8_t* x0[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int m = mt * 8 + g;
    x0[mt] = xs + (size_t)(m < p.M ? m : 0) * p.row_stride + t * 32 + (2 * g_lo) * 128;
  }
  const uint8_t* slot0 = ring + lane * 16;

  for (int r = 0; r < rounds; ++r) {
    float acc[MT][4], acc_u[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][i] = acc_u[mt][i] = 0.f;
    const bool active = r < my_rounds;
    const int band = band_lo + wi + r * p.wn;
    if (active) {
      for (int bb = 0; bb < nbp; ++bb) {
        const uint8_t* xb[MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) xb[mt] = x0[mt] + bb * D * 256;
#pragma unroll
        for (int k = 0; k < D; ++k) {
          cpa_wait<D - 1>();          // this lane's bytes of group bb * D + k have landed
          if (bb * D + k < ng) {      // else padding: nothing was copied, nothing to add
            const uint8_t* st = slot0 + k * kSB;
            GroupWords cur;
            cur.w0 = *reinterpret_cast<const uint4*>(st);
            cur.w1 = *reinterpret_cast<const uint4*>(st + kTileBytes);
            const uint8_t* xg[MT];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) xg[mt] = xb[mt] + k * 256;
            if (FMT == kFmtFp8) {
              group_fp8<MT>(st, xg, acc);
              if (FUSE) group_fp8<MT>(st + kSB1, xg, acc_u);
            } else if (FMT == 0) {
              cur.s0.x = *reinterpret_cast<const uint32_t*>(st + kGroupBytes - lane * 12);
              group_int4<MT>(cur, xg, acc);
            } else {
              const uint4 sv = *reinterpret_cast<const uint4*>(st + kGroupBytes);
              cur.s0 = make_uint2(sv.x, sv.y);
              cur.s1 = make_uint2(sv.z, sv.w);
              block_nvfp4<MT>(cur.w0, cur.s0, xg, acc);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) xg[mt] += 128;
              block_nvfp4<MT>(cur.w1, cur.s1, xg, acc);
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) xg[mt] -= 128;
            }
            if (FUSE && FMT != kFmtFp8) {   // the up band's group, same activations
              const uint8_t* su = st + kSB1;
              GroupWords up;
              up.w0 = *reinterpret_cast<const uint4*>(su);
              up.w1 = *reinterpret_cast<const uint4*>(su + kTileBytes);
              if (FMT == 0) {
                up.s0.x = *reinterpret_cast<const uint32_t*>(su + kGroupBytes - lane * 12);
                group_int4<MT>(up, xg, acc_u);
              } else {
                const uint4 sv = *reinterpret_cast<const uint4*>(su + kGroupBytes);
                block_nvfp4<MT>(up.w0, make_uint2(sv.x, sv.y), xg, acc_u);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) xg[mt] += 128;
                block_nvfp4<MT>(up.w1, make_uint2(sv.z, sv.w), xg, acc_u);
              }
            }
          }
          copy_item(k);               // refill the slot just read
        }
        next_block();
      }
    }
    if (p.wk_log2 == 0) {
      if (active) band_epilogue<FMT, MT, FUSE>(p, band, split, lane, row_mul, acc, acc_u);
      continue;
    }
    // add the wk pieces of each band in piece order
    constexpr int kLaneFloats = 4 * MT * (FUSE ? 2 : 1);
    float* mine = red + (warp * 32 + lane) * kLaneFloats;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mine[mt * 4 + i] = active ? acc[mt][i] : 0.f;
        if (FUSE) mine[4 * MT + mt * 4 + i] = active ? acc_u[mt][i] : 0.f;
      }
    __syncthreads();
    if (wj == 0 && active) {
      float sum[MT][4], sum_u[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sum[mt][i] = sum_u[mt][i] = 0.f;
      for (int pc = 0; pc < (1 << p.wk_log2); ++pc) {
        const float* o = red + ((pc * p.wn + wi) * 32 + lane) * kLaneFloats;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            sum[mt][i] += o[mt * 4 + i];
            if (FUSE) sum_u[mt][i] += o[4 * MT + mt * 4 + i];
          }
      }
      band_epilogue<FMT, MT, FUSE>(p, band, split, lane, row_mul, sum, sum_u);
    }
    __syncthreads();
  }
  cpa_wait<0>();  // nothing is in flight at exit
  if (!x_ok) mbar_wait(xbar, 0, p.err);   // the activation copy, if it ever lands
}

// Raise the dynamic shared memory limit of one kernel variant, once per
// device (kept out of the steady state).  Two host threads may both set it the
// first time; the attribute call is idempotent and the flag is atomic.
template <int FMT, int MT, int D, bool FUSE>
cudaError_t prepare_d(int dev) {
  static std::atomic<bool> smem_set[64];
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!smem_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<FMT, MT, D, FUSE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    smem_set[dev].store(true, std::memory_order_release);
  }
  return cudaSuccess;
}

template <int FMT, int MT, int D, bool FUSE>
cudaError_t launch_d(const Params& p, const GemvPlan& pl, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = prepare_d<FMT, MT, D, FUSE>(dev)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.ctas_x, pl.S);
  cfg.blockDim = dim3(Cfg<FMT, MT, FUSE>::kWarps * 32);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<FMT, MT, D, FUSE>, p);
}

int ilog2(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

template <int FMT, int MT, bool FUSE>
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
  p.I = a.N / 2;
  p.NT = FUSE ? p.I / 16 : (a.N + 15) / 16;    // fused: bands of gate rows
  const size_t KB = (size_t)a.K / 64;
  p.up_w = (size_t)(p.I / 16) * KB * (FMT == kFmtFp8 ? 2 : 1) * kTileBytes;
  p.up_s = FMT == 0 ? (size_t)(p.I / 16) * (a.K / 128) * 32
           : FMT == 1 ? (size_t)(p.I / 16) * KB * 64 : 0;
  p.S = pl.S;
  p.kslice = pl.kslice;
  p.bq = p.NT / pl.ctas_x;
  p.br = p.NT % pl.ctas_x;
  p.row_stride = (pl.kslice / 64) * 128 + 16;
  // staging threads per row: the CTA's threads over M rounded up to a power of two
  p.stage_log2 = ilog2(Cfg<FMT, MT, FUSE>::kWarps * 32) - ilog2(a.M);
  p.wn = pl.wn;
  p.wn_log2 = ilog2(pl.wn);
  p.wk_log2 = ilog2(pl.wk);
  p.ngp = pl.ngp;
  if constexpr (FUSE || FMT == kFmtFp8) {       // stages two or four times as large: D <= 4
    switch (pl.depth) {
      case 2: return launch_d<FMT, MT, 2, FUSE>(p, pl, st);
      case 3: return launch_d<FMT, MT, 3, FUSE>(p, pl, st);
      default: return launch_d<FMT, MT, 4, FUSE>(p, pl, st);
    }
  } else {
    switch (pl.depth) {
      case 2: return launch_d<FMT, MT, 2, FUSE>(p, pl, st);
      case 3: return launch_d<FMT, MT, 3, FUSE>(p, pl, st);
      case 4: return launch_d<FMT, MT, 4, FUSE>(p, pl, st);
      case 5: return launch_d<FMT, MT, 5, FUSE>(p, pl, st);
      case 6: return launch_d<FMT, MT, 6, FUSE>(p, pl, st);
      default: return launch_d<FMT, MT, 8, FUSE>(p, pl, st);
    }
  }
}

// Shared-memory bytes of the FP16 activation image of M rows and `groups`
// 128-groups (one 16-byte pad per row).
int image_bytes(int M, int groups) { return M * (groups * 256 + 16); }

int warps_of(int fmt, int mt) {
  if (fmt == 0) return mt == 1 ? Cfg<0, 1>::kWarps : Cfg<0, 2>::kWarps;
  return mt == 1 ? Cfg<1, 1>::kWarps : Cfg<1, 2>::kWarps;
}

int header_of(int fmt, int mt, int fuse) {
  (void)fmt;   // the header depends on the row tiles and fusion only
  if (fuse) return mt == 1 ? Cfg<0, 1, true>::kHeader : Cfg<0, 2, true>::kHeader;
  return mt == 1 ? Cfg<0, 1>::kHeader : Cfg<0, 2>::kHeader;
}

// Every ring depth a plan can pick for one (format, row tiles, fusion).
template <int FMT, int MT, bool FUSE>
cudaError_t prepare_t(int dev) {
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = prepare_d<FMT, MT, 2, FUSE>(dev);
  if (e == cudaSuccess) e = prepare_d<FMT, MT, 3, FUSE>(dev);
  if (e == cudaSuccess) e = prepare_d<FMT, MT, 4, FUSE>(dev);
  if constexpr (!FUSE && FMT != kFmtFp8) {
    if (e == cudaSuccess) e = prepare_d<FMT, MT, 5, FUSE>(dev);
    if (e == cudaSuccess) e = prepare_d<FMT, MT, 6, FUSE>(dev);
    if (e == cudaSuccess) e = prepare_d<FMT, MT, 8, FUSE>(dev);
  }
  return e;
}

}  // namespace

cudaError_t gemv_prepare_all(int fuse) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const cudaError_t r[6] = {
      fuse ? prepare_t<0, 1, true>(dev) : prepare_t<0, 1, false>(dev),
      fuse ? prepare_t<0, 2, true>(dev) : prepare_t<0, 2, false>(dev),
      fuse ? prepare_t<1, 1, true>(dev) : prepare_t<1, 1, false>(dev),
      fuse ? prepare_t<1, 2, true>(dev) : prepare_t<1, 2, false>(dev),
      fuse ? prepare_t<2, 1, true>(dev) : prepare_t<2, 1, false>(dev),
      fuse ? prepare_t<2, 2, true>(dev) : prepare_t<2, 2, false>(dev)};
  for (cudaError_t x : r)
    if (x != cudaSuccess) return x;
  return cudaSuccess;
}

// Picks the K splits across CTAs (S), the warp grid (wn bands x wk pieces,
// both powers of two) and the ring depth D.  Every warp's piece is padded to
// a multiple of D groups (padding groups copy and add nothing) so that ring
// slots stay compile-time constants across bands.  The cost is the largest
// number of 64-blocks any warp processes (padding included) plus one per
// round, 3 + S/2 for a cross-CTA split and a little for shallow rings; its
// constants were fitted to a sweep of (S, wk, D) over the decode shapes at
// M = 1, 4 and 8 on B200.  The activation image and the rings must fit in
// shared memory together.
GemvPlan plan_gemv(int fmt, int M, int N, int K, int num_sms, int fuse) {
  GemvPlan pl;
  pl.mt = M <= 8 ? 1 : 2;
  const int warps = warps_of(fmt, pl.mt);
  const int header = header_of(fmt, pl.mt, fuse);
  const int sb = stage_bytes(fmt) * (fuse ? 2 : 1);   // fused: gate and up group per stage
  const int NT = fuse ? N / 32 : (N + 15) / 16;       // fused: bands of the I gate rows
  const int depth_cap = (fuse || fmt == kFmtFp8) ? 4 : kMaxDepth;
  // cost per group in units of one 4-bit band-group (1 KB): x2 fused, x2 FP8
  const double per_group = 2.0 * (fuse ? 2 : 1) * (fmt == kFmtFp8 ? 2 : 1);
  const int groups = K / 128;
  double best = 1e300;
  pl.S = 0;
  static const int kSplits[] = {1, 2, 3, 4, 6, 8, 12, 16, 24, 32};
  for (int S : kSplits) {
    if (S > groups) break;
    const int gslice = (groups + S - 1) / S;
    if ((S - 1) * gslice >= groups) continue;  // an empty split
    const int ximg = image_bytes(M, gslice);
    const int dmax = min(depth_cap, (kMaxSmem - header - ximg) / (warps * sb));
    if (dmax < 2) continue;
    int ctas = num_sms / S;
    if (ctas < 1) ctas = 1;
    if (ctas > NT) ctas = NT;
    const int bands_max = (NT + ctas - 1) / ctas;
    for (int wk = 1; wk <= warps; wk *= 2) {
      if (wk > gslice) break;
      const int wn = warps / wk;
      const int rounds = (bands_max + wn - 1) / wn;
      const int piece = (gslice + wk - 1) / wk;
      for (int d = 2; d <= dmax; ++d) {
        if (d == 7) continue;                  // not instantiated
        const int padded = (piece + d - 1) / d * d;
        // plain layers: padding groups copy nothing, so they cost loop
        // overhead rather than bytes, and a ring shallower than 4 costs in
        // proportion to the group's bytes (FP8: measured 8.6 -> 7.8 us on
        // QKV at M = 1 with 4 stages instead of 2); the fused layer keeps
        // the fit it was measured with
        const double pad_cost = fuse ? per_group : 0.5;
        const double shallow = fuse ? 0.5 : 0.25 * per_group;
        double cost = (double)rounds * (per_group * piece + pad_cost * (padded - piece) + 1.0) +
                      (S > 1 ? 3.0 + 0.5 * S : 0.0) + (d < 4 ? shallow * (4 - d) : 0.0);
        // one 8-row tile (M <= 8): + the activation staging, which grows with
        // M x the K slice (a CTA converts its rows' slice before the first
        // MMA), so splitting K pays at M = 4..8 where it does not at M = 1
        // (measured on the O and down projections; at M = 9..16 the fit
        // without it chooses better)
        if (pl.mt == 1) cost += (S > 1 ? 1.34 : 0.0) + 0.0185 * M * gslice;
        if (cost < best - 1e-9) {
          best = cost;
          pl.S = S;
          pl.wk = wk;
          pl.depth = d;
          pl.ngp = padded;
        }
      }
    }
  }
  if (pl.S == 0) {
    // very long K: the smallest split whose activation slice fits
    for (int S = 33; S <= groups && pl.S == 0; ++S) {
      const int gslice = (groups + S - 1) / S;
      if ((S - 1) * gslice >= groups) continue;
      if (kMaxSmem - header - image_bytes(M, gslice) >= warps * 2 * sb) {
        pl.S = S;
        pl.wk = 1;
        pl.depth = 2;
        pl.ngp = (gslice + 1) / 2 * 2;
      }
    }
    if (pl.S == 0) return pl;  // no plan: the caller reports W4A16_ERR_SHAPE
  }
  pl.wn = warps / pl.wk;
  const int gslice = (groups + pl.S - 1) / pl.S;
  pl.kslice = gslice * 128;
  int ctas = num_sms / pl.S;
  if (ctas < 1) ctas = 1;
  if (ctas > NT) ctas = NT;
  pl.ctas_x = ctas;
  pl.smem = header + warps * pl.depth * sb + image_bytes(M, gslice);
  return pl;
}

size_t gemv_workspace_floats(const GemvPlan& p, int M, int N) {
  return p.S > 1 ? static_cast<size_t>(p.S) * M * ((N + 15) / 16 * 16) : 0;
}

size_t gemv_counters(const GemvPlan& p, int N) { return p.S > 1 ? (N + 15) / 16 : 0; }

cudaError_t launch_gemv(const GemvPlan& p, const GemmArgs& a, cudaStream_t st) {
  if (a.fmt == kFmtFp8) {
    if (a.fuse) return p.mt == 1 ? launch_t<2, 1, true>(p, a, st) : launch_t<2, 2, true>(p, a, st);
    return p.mt == 1 ? launch_t<2, 1, false>(p, a, st) : launch_t<2, 2, false>(p, a, st);
  }
  if (a.fuse) {
    if (a.fmt == 0) return p.mt == 1 ? launch_t<0, 1, true>(p, a, st) : launch_t<0, 2, true>(p, a, st);
    return p.mt == 1 ? launch_t<1, 1, true>(p, a, st) : launch_t<1, 2, true>(p, a, st);
  }
  if (a.fmt == 0) return p.mt == 1 ? launch_t<0, 1, false>(p, a, st) : launch_t<0, 2, false>(p, a, st);
  return p.mt == 1 ? launch_t<1, 1, false>(p, a, st) : launch_t<1, 2, false>(p, a, st);
}

}  // namespace w4
