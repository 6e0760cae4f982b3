// Packed weight/scale layout shared by the packers and the kernels.
//
// The weight matrix W[N][K] (output column n, reduction index k) is cut into
// tiles of 16 rows x 64 k.  A tile is 512 bytes, the footprint of one warp's
// 16-byte loads, and tiles of one 16-row band are contiguous along K, so a
// band's K-range is one contiguous byte range (one bulk copy).
//
//   tile (nt, kb), nt = n / 16, kb = k / 64, at byte ((nt * KB) + kb) * 512,
//   KB = K / 64.  Inside a tile, lane L = 4g + t (g = 0..7, t = 0..3) owns the
//   16 bytes at 16 L: four 32-bit words, word j covering k16 sub-block
//   k0 = 64 kb + 16 j.  Each word holds 8 nibbles that form four pairs of
//   adjacent-k elements:
//     P0 = (row g,   k0+4t, k0+4t+1)     P1 = (row g+8, k0+4t, k0+4t+1)
//     P2 = (row g,   k0+4t+2, k0+4t+3)   P3 = (row g+8, k0+4t+2, k0+4t+3)
//   INT4 puts pair p in nibbles p (first element) and p+4 (second), so
//   (word >> 4p) & 0x000F000F drops both into the low bits of a 16-bit half;
//   NVFP4 puts pair p in byte p (first element in the low nibble), the
//   operand order of the hardware e2m1x2 -> f16x2 conversion.
//   The pairs are the operand fragments of both tensor-core paths: the A
//   fragment of mma.sync m16n8k16 (with the k order inside a 16-block
//   permuted, the same permutation applied to the activations) and the
//   register layout of tcgen05.st 16x256b into a K-major TMEM A tile.
//
//   INT4 nibble = q + 8 (offset binary); NVFP4 nibble = e2m1 code.
//   Rows n >= N (padding up to a multiple of 16) hold value 0 and scale 0.
//
// FP8-E4M3 (one byte per weight, one fp32 scale per tensor, no packed
// scales): the same pairs, a byte per element, so a 512-byte tile covers 16
// rows x 32 k.  Tile (nt, kt), kt = k / 32, at ((nt * K/32) + kt) * 512; lane
// L = 4g + t owns the 16 bytes at 16 L: for k16 sub-block j (0, 1) of the
// tile, word 2j holds P0 (bytes 0, 1) and P1 (bytes 2, 3), word 2j + 1 holds
// P2 and P3, first element in the lower byte: the operand order of the
// hardware e4m3x2 -> f16x2 conversion.  A 128-group of a band is four tiles.
//
// Scales:
//   INT4: per (nt, group gi = k / 128), 32 bytes at (nt * (K/128) + gi) * 32;
//         BF16 of row nt*16 + g + 8h at byte 4g + 2h (h = 0, 1), so lane
//         (g, t) reads the scales of its rows g and g+8 with one 32-bit load.
//   NVFP4: per (nt, kb), 64 bytes at (nt * KB + kb) * 64; E4M3 of row
//         nt*16 + g + 8h, group 4 kb + j at byte 8g + 2j + h.
#pragma once

#include <stdint.h>
#include <stddef.h>

#ifdef __CUDACC__
#define W4_HD __host__ __device__ __forceinline__
#else
#define W4_HD inline
#endif

namespace w4 {

constexpr int kTileRows = 16;
constexpr int kTileK = 64;
constexpr int kTileBytes = 512;
constexpr int kInt4Group = 128;
constexpr int kNvfp4Group = 16;
constexpr int kInt4ScaleBlockBytes = 32;   // per (nt, 128-group)
constexpr int kNvfp4ScaleBlockBytes = 64;  // per (nt, k64 block)
constexpr int kFmtFp8 = 2;                 // FP8-E4M3 weights, per-tensor fp32 scale

W4_HD int64_t padded_rows(int64_t N) { return (N + 15) / 16 * 16; }

W4_HD int64_t weight_bytes(int fmt, int64_t N, int64_t K) {
  return fmt == kFmtFp8 ? padded_rows(N) * K : padded_rows(N) * K / 2;
}

W4_HD int64_t scale_bytes(int fmt, int64_t N, int64_t K) {
  if (fmt == kFmtFp8) return 0;
  return fmt == 0 ? padded_rows(N) * (K / kInt4Group) * 2 : padded_rows(N) * (K / kNvfp4Group);
}

// Byte offset of element (n, k) in packed FP8-E4M3 weights.
W4_HD int64_t fp8_pos(int64_t n, int64_t k, int64_t K) {
  const int64_t nt = n >> 4, kt = k >> 5;
  const int r = (int)(n & 15), kk = (int)(k & 31);
  const int g = r & 7, hi_row = r >> 3;
  const int j = kk >> 4, kin = kk & 15;
  const int t = kin >> 2, e = kin & 3;
  const int pair = hi_row + 2 * (e >> 1);        // P0..P3
  const int second = e & 1;
  const int word = 2 * j + (pair >> 1);
  return ((nt * (K >> 5) + kt) * 512) + (4 * g + t) * 16 + word * 4 + 2 * (pair & 1) + second;
}

// Position of element (n, k) in the packed weights: byte offset and nibble
// shift (0 = low nibble of that byte).
struct NibblePos {
  int64_t byte;
  int shift;
};

W4_HD NibblePos weight_pos(int fmt, int64_t n, int64_t k, int64_t K) {
  const int64_t nt = n >> 4, kb = k >> 6;
  const int r = (int)(n & 15), kk = (int)(k & 63);
  const int g = r & 7, hi_row = r >> 3;          // row g or g+8
  const int j = kk >> 4, kin = kk & 15;
  const int t = kin >> 2, e = kin & 3;           // k0 + 4t + e
  const int pair = hi_row + 2 * (e >> 1);        // P0..P3
  const int second = e & 1;                      // first or second element of the pair
  const int nib = fmt == 0 ? pair + 4 * second : 2 * pair + second;
  const int64_t word = ((nt * (K >> 6) + kb) * 512) + (4 * g + t) * 16 + j * 4;
  NibblePos p;
  p.byte = word + (nib >> 1);
  p.shift = (nib & 1) * 4;
  return p;
}

W4_HD int64_t int4_scale_offset(int64_t n, int64_t gi, int64_t K) {
  const int64_t nt = n >> 4;
  const int r = (int)(n & 15);
  return (nt * (K / kInt4Group) + gi) * 32 + (r & 7) * 4 + (r >> 3) * 2;
}

W4_HD int64_t nvfp4_scale_offset(int64_t n, int64_t gi, int64_t K) {
  const int64_t nt = n >> 4, kb = gi >> 2;
  const int r = (int)(n & 15), j = (int)(gi & 3);
  return (nt * (K >> 6) + kb) * 64 + (r & 7) * 8 + j * 2 + (r >> 3);
}

}  // namespace w4
