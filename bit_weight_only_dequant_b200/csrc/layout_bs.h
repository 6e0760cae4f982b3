// Packed layout of NVFP4 weights for the W4A4 block-scaled tensor-core path
// (format id 3, W4A16_FMT_NVFP4_BS): the operand layout of tcgen05.mma
// kind::mxf4nvf4 as the tensor memory accelerator (TMA) and the 32x128b
// tensor-memory copy read it, so that the kernel streams it without touching
// a value.
//
//  * Codes: [N][K/2] bytes, row-major; byte j of row n holds k = 2j in its low
//    nibble and k = 2j + 1 in its high nibble (E2M1, bit 3 the sign).  No row
//    padding: the TMA load of a 128-row tile fills rows past N with zero.
//  * Scales: one E4M3 byte per (row, 16-k block), in atoms of 128 rows x 64 k
//    (512 bytes): atom (t, kb) of row tile t = n / 128 and 64-k block kb
//    holds row n = 128 t + a + 32 b, 16-block j of kb at byte 16 a + 4 b + j.
//    Atoms are ordered (t, kb), so the four atoms of a 256-k stage are 2 KB
//    of consecutive bytes; rows of the last tile past N hold scale 0.
// The activations of the W4A4 matmul use the same two layouts ([M][K/2]
// codes; atoms per chunk of at most 128 rows), written by the quantiser.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define W4BS_HD __host__ __device__ __forceinline__
#else
#define W4BS_HD inline
#endif

namespace w4 {

constexpr int kFmtNvfp4Bs = 3;
constexpr int kBsTileRows = 128;     // rows of a scale atom and of the MMA's M
constexpr int kBsAtomBytes = 512;    // 128 rows x 4 scale bytes (64 k)

W4BS_HD int64_t bs_tiles(int64_t N) { return (N + kBsTileRows - 1) / kBsTileRows; }

W4BS_HD int64_t bs_weight_bytes(int64_t N, int64_t K) { return N * K / 2; }

W4BS_HD int64_t bs_scale_bytes(int64_t N, int64_t K) { return bs_tiles(N) * (K / 64) * kBsAtomBytes; }

// Byte of the scale of row r (within its 128-row tile or chunk `t`) and
// 16-block gi, in a run of atoms with K/64 atoms per tile.
W4BS_HD int64_t bs_scale_offset(int64_t t, int r, int64_t gi, int64_t K) {
  return (t * (K >> 6) + (gi >> 2)) * kBsAtomBytes + (r & 31) * 16 + (r >> 5) * 4 + (gi & 3);
}

}  // namespace w4
