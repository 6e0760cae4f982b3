// Packers between the logical checkpoint tensors and the library layout
// (layout.h): a host version with range checks, its inverse, and a device
// version for packing large matrices where they already live.
#include <string.h>

#include "bs.h"
#include "common.cuh"
#include "kernels.h"

namespace w4 {

// ---------------------------------------------------------------- host

int pack_host(int fmt, int N, int K, const void* codes_v, const void* scales_v, void* w_v,
              void* s_v) {
  const int64_t Np = padded_rows(N);
  uint8_t* w = static_cast<uint8_t*>(w_v);
  uint8_t* s = static_cast<uint8_t*>(s_v);
  // padding rows: value 0 (int4 nibble 8, e2m1 / e4m3 code 0), scale 0
  memset(w, 0, (size_t)weight_bytes(fmt, N, K));
  if (fmt == kFmtFp8) {
    const uint8_t* c = static_cast<const uint8_t*>(codes_v);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) {
        const uint8_t b = c[n * K + k];
        if ((b & 0x7Fu) == 0x7Fu) return -1;  // E4M3 NaN
        w[fp8_pos(n, k, K)] = b;
      }
    return 0;
  }
  memset(s, 0, (size_t)scale_bytes(fmt, N, K));
  if (fmt == 0) {
    const int8_t* q = static_cast<const int8_t*>(codes_v);
    for (int64_t n = 0; n < Np; ++n) {
      for (int64_t k = 0; k < K; ++k) {
        int v = 0;
        if (n < N) {
          v = q[n * K + k];
          if (v < -8 || v > 7) return -1;
        }
        const NibblePos pos = weight_pos(0, n, k, K);
        w[pos.byte] |= static_cast<uint8_t>((v + 8) << pos.shift);
      }
    }
    const uint16_t* sc = static_cast<const uint16_t*>(scales_v);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t gi = 0; gi < K / kInt4Group; ++gi) {
        const uint16_t b = sc[n * (K / kInt4Group) + gi];
        if ((b & 0x7F80u) == 0x7F80u) return -1;  // inf / NaN scale
        memcpy(s + int4_scale_offset(n, gi, K), &b, 2);
      }
  } else {
    const uint8_t* c = static_cast<const uint8_t*>(codes_v);
    for (int64_t n = 0; n < N; ++n) {
      for (int64_t k = 0; k < K; ++k) {
        const int v = c[n * K + k];
        if (v > 15) return -1;
        const NibblePos pos = weight_pos(1, n, k, K);
        w[pos.byte] |= static_cast<uint8_t>(v << pos.shift);
      }
    }
    const uint8_t* sc = static_cast<const uint8_t*>(scales_v);
    for (int64_t n = 0; n < N; ++n)
      for (int64_t gi = 0; gi < K / kNvfp4Group; ++gi) {
        const uint8_t b = sc[n * (K / kNvfp4Group) + gi];
        if ((b & 0x7Fu) == 0x7Fu) return -1;  // E4M3 NaN
        s[nvfp4_scale_offset(n, gi, K)] = b;
      }
  }
  return 0;
}

int unpack_host(int fmt, int N, int K, const void* w_v, const void* s_v, void* codes_v,
                void* scales_v) {
  const uint8_t* w = static_cast<const uint8_t*>(w_v);
  const uint8_t* s = static_cast<const uint8_t*>(s_v);
  if (fmt == kFmtFp8) {
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k)
        static_cast<uint8_t*>(codes_v)[n * K + k] = w[fp8_pos(n, k, K)];
    return 0;
  }
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      const NibblePos pos = weight_pos(fmt, n, k, K);
      const int v = (w[pos.byte] >> pos.shift) & 15;
      if (fmt == 0)
        static_cast<int8_t*>(codes_v)[n * K + k] = static_cast<int8_t>(v - 8);
      else
        static_cast<uint8_t*>(codes_v)[n * K + k] = static_cast<uint8_t>(v);
    }
  if (fmt == 0) {
    for (int64_t n = 0; n < N; ++n)
      for (int64_t gi = 0; gi < K / kInt4Group; ++gi)
        memcpy(static_cast<uint16_t*>(scales_v) + n * (K / kInt4Group) + gi,
               s + int4_scale_offset(n, gi, K), 2);
  } else {
    for (int64_t n = 0; n < N; ++n)
      for (int64_t gi = 0; gi < K / kNvfp4Group; ++gi)
        static_cast<uint8_t*>(scales_v)[n * (K / kNvfp4Group) + gi] =
            s[nvfp4_scale_offset(n, gi, K)];
  }
  return 0;
}

// ---------------------------------------------------------------- device

namespace {

// One thread per (tile, lane): gathers its 32 codes and writes 16 bytes.
template <int FMT>
__global__ void pack_weights_kernel(int N, int K, const uint8_t* __restrict__ codes,
                                    uint8_t* __restrict__ w) {
  const int KB = K >> 6;
  const long long total = (long long)((N + 15) / 16) * KB * 32;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int lane = (int)(idx & 31);
    const long long tile = idx >> 5;
    const long long nt = tile / KB;
    const int kb = (int)(tile - nt * KB);
    const int g = lane >> 2, t = lane & 3;
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int hrow = 0; hrow < 2; ++hrow) {
        const long long n = nt * 16 + g + 8 * hrow;
        const int k0 = kb * 64 + j * 16 + 4 * t;
        uint32_t u[4] = {FMT == 0 ? 8u : 0u, FMT == 0 ? 8u : 0u, FMT == 0 ? 8u : 0u,
                         FMT == 0 ? 8u : 0u};
        if (n < N) {
          const uint32_t four = *reinterpret_cast<const uint32_t*>(codes + n * (long long)K + k0);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t b = (four >> (8 * e)) & 0xFFu;
            u[e] = FMT == 0 ? ((b + 8u) & 15u) : (b & 15u);  // int8 q -> q + 8
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pair = hrow + 2 * (e >> 1), second = e & 1;
          const int nib = FMT == 0 ? pair + 4 * second : 2 * pair + second;
          wd[j] |= u[e] << (4 * nib);
        }
      }
    }
    *reinterpret_cast<uint4*>(w + tile * kTileBytes + lane * 16) =
        make_uint4(wd[0], wd[1], wd[2], wd[3]);
  }
}

// FP8: one thread per (32-k tile, lane), 16 codes of its two rows.
__global__ void pack_fp8_kernel(int N, int K, const uint8_t* __restrict__ codes,
                                uint8_t* __restrict__ w) {
  const int KT = K >> 5;
  const long long total = (long long)((N + 15) / 16) * KT * 32;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int lane = (int)(idx & 31);
    const long long tile = idx >> 5;
    const long long nt = tile / KT;
    const int kt = (int)(tile - nt * KT);
    const int g = lane >> 2, t = lane & 3;
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int hrow = 0; hrow < 2; ++hrow) {
        const long long n = nt * 16 + g + 8 * hrow;
        const int k0 = kt * 32 + j * 16 + 4 * t;
        const uint32_t four =
            n < N ? *reinterpret_cast<const uint32_t*>(codes + n * (long long)K + k0) : 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pair = hrow + 2 * (e >> 1), second = e & 1;
          const int byte = 2 * (pair & 1) + second;
          wd[2 * j + (pair >> 1)] |= ((four >> (8 * e)) & 0xFFu) << (8 * byte);
        }
      }
    }
    *reinterpret_cast<uint4*>(w + tile * kTileBytes + lane * 16) =
        make_uint4(wd[0], wd[1], wd[2], wd[3]);
  }
}

template <int FMT>
__global__ void pack_scales_kernel(int N, int K, const uint8_t* __restrict__ scales,
                                   uint8_t* __restrict__ s) {
  const int G = FMT == 0 ? K / kInt4Group : K / kNvfp4Group;
  const long long Np = (N + 15) / 16 * 16;
  const long long total = Np * G;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long n = idx / G;
    const int gi = (int)(idx - n * G);
    if (FMT == 0) {
      const uint16_t v = n < N ? reinterpret_cast<const uint16_t*>(scales)[n * G + gi] : 0;
      *reinterpret_cast<uint16_t*>(s + int4_scale_offset(n, gi, K)) = v;
    } else {
      s[nvfp4_scale_offset(n, gi, K)] = n < N ? scales[n * G + gi] : 0;
    }
  }
}

}  // namespace

cudaError_t launch_pack(int fmt, int N, int K, const void* codes, const void* scales, void* w,
                        void* s, cudaStream_t st) {
  if (fmt == kFmtFp8) {
    const long long ft = (long long)((N + 15) / 16) * (K / 32) * 32;
    const unsigned bf = (unsigned)((ft + 255) / 256 < 148 * 32 ? (ft + 255) / 256 : 148 * 32);
    pack_fp8_kernel<<<bf, 256, 0, st>>>(N, K, (const uint8_t*)codes, (uint8_t*)w);
    return cudaGetLastError();
  }
  const long long wt = (long long)((N + 15) / 16) * (K / 64) * 32;
  const long long sc = (long long)((N + 15) / 16 * 16) * (fmt == 0 ? K / 128 : K / 16);
  const unsigned bw = (unsigned)((wt + 255) / 256 < 148 * 32 ? (wt + 255) / 256 : 148 * 32);
  const unsigned bs = (unsigned)((sc + 255) / 256 < 148 * 32 ? (sc + 255) / 256 : 148 * 32);
  if (fmt == 0) {
    pack_weights_kernel<0><<<bw, 256, 0, st>>>(N, K, (const uint8_t*)codes, (uint8_t*)w);
    pack_scales_kernel<0><<<bs, 256, 0, st>>>(N, K, (const uint8_t*)scales, (uint8_t*)s);
  } else {
    pack_weights_kernel<1><<<bw, 256, 0, st>>>(N, K, (const uint8_t*)codes, (uint8_t*)w);
    pack_scales_kernel<1><<<bs, 256, 0, st>>>(N, K, (const uint8_t*)scales, (uint8_t*)s);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- block-scaled W4A4 layout

int pack_host_bs(int N, int K, const void* codes_v, const void* scales_v, void* w_v, void* s_v) {
  const uint8_t* c = static_cast<const uint8_t*>(codes_v);
  const uint8_t* sc = static_cast<const uint8_t*>(scales_v);
  uint8_t* w = static_cast<uint8_t*>(w_v);
  uint8_t* s = static_cast<uint8_t*>(s_v);
  memset(s, 0, (size_t)bs_scale_bytes(N, K));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 2; ++j) {
      const uint8_t lo = c[n * K + 2 * j], hi = c[n * K + 2 * j + 1];
      if (lo > 15 || hi > 15) return -1;
      w[n * (K / 2) + j] = static_cast<uint8_t>(lo | (hi << 4));
    }
  for (int64_t n = 0; n < N; ++n)
    for (int64_t gi = 0; gi < K / kNvfp4Group; ++gi) {
      const uint8_t b = sc[n * (K / kNvfp4Group) + gi];
      if ((b & 0x7Fu) == 0x7Fu) return -1;  // E4M3 NaN
      s[bs_scale_offset(n / kBsTileRows, (int)(n % kBsTileRows), gi, K)] = b;
    }
  return 0;
}

int unpack_host_bs(int N, int K, const void* w_v, const void* s_v, void* codes_v, void* scales_v) {
  const uint8_t* w = static_cast<const uint8_t*>(w_v);
  const uint8_t* s = static_cast<const uint8_t*>(s_v);
  uint8_t* c = static_cast<uint8_t*>(codes_v);
  uint8_t* sc = static_cast<uint8_t*>(scales_v);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 2; ++j) {
      const uint8_t b = w[n * (K / 2) + j];
      c[n * K + 2 * j] = b & 15u;
      c[n * K + 2 * j + 1] = b >> 4;
    }
  for (int64_t n = 0; n < N; ++n)
    for (int64_t gi = 0; gi < K / kNvfp4Group; ++gi)
      sc[n * (K / kNvfp4Group) + gi] = s[bs_scale_offset(n / kBsTileRows, (int)(n % kBsTileRows), gi, K)];
  return 0;
}

namespace {

// One thread per (row, 16-block) of the padded rows: 8 bytes of codes (rows
// below N) and the block's scale byte (0 past N).
__global__ void pack_bs_kernel(int N, int K, const uint8_t* __restrict__ codes,
                               const uint8_t* __restrict__ scales, uint8_t* __restrict__ w,
                               uint8_t* __restrict__ s) {
  const int G = K / kNvfp4Group;
  const long long total = bs_tiles(N) * kBsTileRows * G;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long n = idx / G;
    const long long gi = idx - n * G;
    uint8_t sv = 0;
    if (n < N) {
      const uint4 v = *reinterpret_cast<const uint4*>(codes + n * K + 16 * gi);
      const uint32_t in[4] = {v.x, v.y, v.z, v.w};
      uint32_t out[2] = {0u, 0u};
#pragma unroll
      for (int j = 0; j < 16; ++j)
        out[j >> 3] |= ((in[j >> 2] >> (8 * (j & 3))) & 15u) << (4 * (j & 7));
      *reinterpret_cast<uint2*>(w + n * (K / 2) + 8 * gi) = make_uint2(out[0], out[1]);
      sv = scales[n * G + gi];
    }
    s[bs_scale_offset(n / kBsTileRows, (int)(n % kBsTileRows), gi, K)] = sv;
  }
}

}  // namespace

cudaError_t launch_pack_bs(int N, int K, const void* codes, const void* scales, void* w, void* s,
                           cudaStream_t st) {
  const long long total = bs_tiles(N) * kBsTileRows * (K / kNvfp4Group);
  const unsigned blocks = (unsigned)((total + 255) / 256 < 148 * 32 ? (total + 255) / 256 : 148 * 32);
  pack_bs_kernel<<<blocks, 256, 0, st>>>(N, K, static_cast<const uint8_t*>(codes),
                                         static_cast<const uint8_t*>(scales),
                                         static_cast<uint8_t*>(w), static_cast<uint8_t*>(s));
  return cudaGetLastError();
}

}  // namespace w4
