"""Seeded synthetic inputs for the W4A16 weight-only matmul.

This module is shared by both sides of every parity check: the fp64 oracle and
the CUDA library each take their inputs from here, and nothing here performs
any of the method's own arithmetic (no dequantisation, no matmul).  It only
draws random numbers and rounds them to their storage types (BF16, FP8-E4M3).

Generator
---------
SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014), used counter-style: element ``i`` of a stream with
key ``key`` is ``mix64(key + (i + 1) * GAMMA)``, i.e. the (i+1)-th output of a
SplitMix64 generator seeded with ``key``.  Streams are keyed by
``(seed, tensor_id)`` through ``stream_key``.  Because every element is a pure
function of its index, any subset of a tensor (one row of a 248,320-row output
projection, say) can be regenerated on its own, and the CUDA twin in
``synth/csrc/synth_gen.cu`` reproduces the same values on the device.

Draws
-----
* 4-bit codes: the top 4 bits of the 64-bit output (exactly uniform on 0..15).
* uniform double in (0, 1): ``((z >> 11) + 0.5) * 2**-53``.
* standard normal: Box-Muller on the uniforms of counters ``2i`` and ``2i+1``,
  ``sqrt(-2 ln u1) * cos(2 pi u2)`` (the sine half is not used).

Value recipes (the workload of the 5120-hidden dense model's linears)
--------------------------------------------------------------------
* int4 GPTQ weights: q = code - 8, uniform on [-8, 7].
* int4 group scales (one per 128 K-elements per output column):
  RNE_bf16(0.01 * exp(0.25 * z)), z ~ N(0, 1); 0.25 is read as the standard
  deviation of the log-normal exponent.
* activations: RNE_bf16(z), z ~ N(0, 1).
* NVFP4 e2m1 codes: uniform on the 16 codes.
* NVFP4 group scales (one per 16 K-elements per output column):
  RNE_e4m3(|z| * 0.05), saturating at 448.
* NVFP4 per-tensor scale: fp32(1/448).
* FP8-E4M3 weights (W8A16): sign(z) * RNE_e4m3(|z| * 64), z ~ N(0, 1), with
  the per-tensor scale fp32(1/448).  Drawn on the host only (no CUDA twin);
  ``device_problem`` copies them to the device.
"""

from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Tensor ids: one independent stream per logical tensor of a problem.
T_Q = 1        # int4 codes
T_S = 2        # int4 bf16 group scales (normal draws)
T_X = 3        # activations (normal draws)
T_C = 4        # nvfp4 e2m1 codes
T_S8 = 5       # nvfp4 e4m3 group scales (normal draws)
T_W8 = 6       # fp8 e4m3 weights (normal draws)

INT4_GROUP = 128
NVFP4_GROUP = 16


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function (the 'mix' finaliser), on uint64 arrays."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    """Key of the stream for one tensor of one seeded problem."""
    with np.errstate(over="ignore"):
        a = mix64(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + GAMMA)
        b = mix64(a + np.uint64(tensor_id) * GAMMA)
    return np.uint64(b)


def raw64(seed: int, tensor_id: int, index: np.ndarray) -> np.ndarray:
    """64-bit outputs for the given element indices of one stream."""
    key = stream_key(seed, tensor_id)
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(key + (idx + np.uint64(1)) * GAMMA)


def codes4(seed: int, tensor_id: int, index: np.ndarray) -> np.ndarray:
    """Uniform 4-bit codes (0..15) from the top bits."""
    return (raw64(seed, tensor_id, index) >> np.uint64(60)).astype(np.uint8)


def _unit(z: np.ndarray) -> np.ndarray:
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normals(seed: int, tensor_id: int, index: np.ndarray) -> np.ndarray:
    """Standard normals (float64) by Box-Muller on counters 2i and 2i+1."""
    idx = np.asarray(index, dtype=np.uint64)
    u1 = _unit(raw64(seed, tensor_id, idx * np.uint64(2)))
    u2 = _unit(raw64(seed, tensor_id, idx * np.uint64(2) + np.uint64(1)))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


# ---------------------------------------------------------------- rounding to storage types


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values to BF16 (round to nearest, ties to even); uint16 bits.

    Normal range: keep 8 significant bits of the binary mantissa from frexp;
    BF16 subnormal range (below 2**-126): quantum 2**-133.  Values here stay
    far from overflow.
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    small = np.abs(v) < 2.0 ** -126
    r = np.where(small, np.ldexp(np.rint(np.ldexp(v, 133)), -133), r)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def to_e4m3_bytes(v: np.ndarray) -> np.ndarray:
    """Round non-negative float64 values to OCP FP8-E4M3 (RNE, saturating at 448)."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(~np.isfinite(v)):
        raise ValueError("e4m3 scale draws must be finite and non-negative")
    m, e = np.frexp(v)
    r = np.ldexp(np.rint(np.ldexp(m, 4)), e - 4)          # 4 significant bits
    sub = v < 2.0 ** -6
    r = np.where(sub, np.ldexp(np.rint(np.ldexp(v, 9)), -9), r)  # quantum 2**-9
    r = np.minimum(r, 448.0)
    out = np.zeros(v.shape, dtype=np.uint8)
    nz = r > 0
    is_sub = nz & (r < 2.0 ** -6)
    out[is_sub] = np.ldexp(r[is_sub], 9).astype(np.uint8)
    nrm = nz & ~is_sub
    mm, ee = np.frexp(r[nrm])                              # r = mm * 2**ee, mm in [0.5, 1)
    field = (ee - 1 + 7).astype(np.int64)
    mant = (np.ldexp(mm, 4) - 8).astype(np.int64)          # 3 fraction bits
    out[nrm] = ((field << 3) | mant).astype(np.uint8)
    return out


# ---------------------------------------------------------------- problem tensors


def int4_weights(seed: int, N: int, K: int, rows=None) -> np.ndarray:
    """q[n][k] as int8 in [-8, 7]; ``rows`` selects a subset of output columns n."""
    rows = np.arange(N, dtype=np.uint64) if rows is None else np.asarray(rows, dtype=np.uint64)
    idx = rows[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :]
    return (codes4(seed, T_Q, idx).astype(np.int16) - 8).astype(np.int8)


def int4_scales(seed: int, N: int, K: int, rows=None) -> np.ndarray:
    """BF16 bits of the per-(column, 128-group) scales, shape [len(rows)][K/128]."""
    G = K // INT4_GROUP
    rows = np.arange(N, dtype=np.uint64) if rows is None else np.asarray(rows, dtype=np.uint64)
    idx = rows[:, None] * np.uint64(G) + np.arange(G, dtype=np.uint64)[None, :]
    return to_bf16_bits(0.01 * np.exp(0.25 * normals(seed, T_S, idx)))


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """BF16 bits of x[m][k] ~ N(0, 1), shape [M][K]."""
    idx = np.arange(M * K, dtype=np.uint64).reshape(M, K)
    return to_bf16_bits(normals(seed, T_X, idx))


def nvfp4_codes(seed: int, N: int, K: int, rows=None) -> np.ndarray:
    rows = np.arange(N, dtype=np.uint64) if rows is None else np.asarray(rows, dtype=np.uint64)
    idx = rows[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :]
    return codes4(seed, T_C, idx)


def nvfp4_scales(seed: int, N: int, K: int, rows=None) -> np.ndarray:
    """E4M3 bytes of the per-(column, 16-group) scales, shape [len(rows)][K/16]."""
    G = K // NVFP4_GROUP
    rows = np.arange(N, dtype=np.uint64) if rows is None else np.asarray(rows, dtype=np.uint64)
    idx = rows[:, None] * np.uint64(G) + np.arange(G, dtype=np.uint64)[None, :]
    return to_e4m3_bytes(np.abs(normals(seed, T_S8, idx)) * 0.05)


NVFP4_GLOBAL_SCALE = float(np.float32(1.0 / 448.0))
FP8_GLOBAL_SCALE = float(np.float32(1.0 / 448.0))


def fp8_weights(seed: int, N: int, K: int, rows=None) -> np.ndarray:
    """E4M3 bytes of the weights [len(rows)][K]: sign(z) * RNE_e4m3(|z| * 64)."""
    rows = np.arange(N, dtype=np.uint64) if rows is None else np.asarray(rows, dtype=np.uint64)
    idx = rows[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :]
    z = normals(seed, T_W8, idx)
    return to_e4m3_bytes(np.abs(z) * 64.0) | np.where(z < 0, 0x80, 0).astype(np.uint8)


def problem(fmt: str, seed: int, M: int, N: int, K: int, rows=None) -> dict:
    """All logical tensors of one seeded problem (host numpy arrays).

    fmt: "int4" or "nvfp4".  Returns codes/scales/x (+ g for nvfp4).  The
    activations of a problem are keyed by the same seed as its weights.
    """
    if fmt == "int4":
        return {"fmt": fmt, "M": M, "N": N, "K": K,
                "codes": int4_weights(seed, N, K, rows),
                "scales": int4_scales(seed, N, K, rows),
                "x": activations(seed, M, K), "g": None}
    if fmt == "nvfp4":
        return {"fmt": fmt, "M": M, "N": N, "K": K,
                "codes": nvfp4_codes(seed, N, K, rows),
                "scales": nvfp4_scales(seed, N, K, rows),
                "x": activations(seed, M, K), "g": NVFP4_GLOBAL_SCALE}
    if fmt == "fp8":
        return {"fmt": fmt, "M": M, "N": N, "K": K,
                "codes": fp8_weights(seed, N, K, rows), "scales": None,
                "x": activations(seed, M, K), "g": FP8_GLOBAL_SCALE}
    raise ValueError(fmt)


# ---------------------------------------------------------------- device twin (CUDA)

import ctypes as _ctypes
import os as _os

_HERE = _os.path.dirname(_os.path.abspath(__file__))
_DEV_LIB_PATH = _os.path.join(_HERE, "libw4a16_synth.so")
_dev_lib = None

KIND_INT4_Q, KIND_INT4_S, KIND_X, KIND_NVFP4_C, KIND_NVFP4_S = 0, 1, 2, 3, 4


def build_device_generator(force: bool = False, verbose: bool = False) -> str:
    """Compile synth/csrc/synth_gen.cu into synth/libw4a16_synth.so (sm_100a)."""
    import shutil
    import subprocess
    src = _os.path.join(_HERE, "csrc", "synth_gen.cu")
    if not force and _os.path.exists(_DEV_LIB_PATH) and \
            _os.path.getmtime(_DEV_LIB_PATH) >= _os.path.getmtime(src):
        return _DEV_LIB_PATH
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-o", _DEV_LIB_PATH, src, "-lcudart"]
    if verbose:
        import sys
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return _DEV_LIB_PATH


def _device_lib():
    global _dev_lib
    if _dev_lib is None:
        if not _os.path.exists(_DEV_LIB_PATH):
            raise RuntimeError(f"{_DEV_LIB_PATH} is missing: run __graft_entry__.build()")
        lib = _ctypes.CDLL(_DEV_LIB_PATH)
        lib.synth_generate.argtypes = [_ctypes.c_int, _ctypes.c_ulonglong, _ctypes.c_int,
                                       _ctypes.c_longlong, _ctypes.c_void_p, _ctypes.c_void_p]
        lib.synth_generate.restype = _ctypes.c_int
        _dev_lib = lib
    return _dev_lib


def device_fill(kind: int, seed: int, tensor_id: int, out, stream=None) -> None:
    """Fill a contiguous torch CUDA tensor with the stream's first numel() draws."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(out.device).cuda_stream
    r = _device_lib().synth_generate(kind, seed & 0xFFFFFFFFFFFFFFFF, tensor_id, out.numel(),
                                     out.data_ptr(), stream)
    if r != 0:
        raise RuntimeError(f"synth_generate failed ({r})")


def device_problem(fmt: str, seed: int, M: int, N: int, K: int, device="cuda"):
    """The tensors of ``problem(fmt, seed, M, N, K)``, drawn on the GPU (torch tensors).

    FP8 weights have no CUDA twin: they are drawn on the host and copied."""
    import torch
    if fmt == "fp8":
        codes = torch.from_numpy(fp8_weights(seed, N, K)).to(device)
        x = torch.empty((M, K), dtype=torch.int16, device=device)
        device_fill(KIND_X, seed, T_X, x)
        return {"fmt": fmt, "M": M, "N": N, "K": K, "codes": codes, "scales": None, "x": x,
                "g": FP8_GLOBAL_SCALE}
    if fmt == "int4":
        codes = torch.empty((N, K), dtype=torch.int8, device=device)
        scales = torch.empty((N, K // INT4_GROUP), dtype=torch.int16, device=device)
        device_fill(KIND_INT4_Q, seed, T_Q, codes)
        device_fill(KIND_INT4_S, seed, T_S, scales)
        g = None
    else:
        codes = torch.empty((N, K), dtype=torch.uint8, device=device)
        scales = torch.empty((N, K // NVFP4_GROUP), dtype=torch.uint8, device=device)
        device_fill(KIND_NVFP4_C, seed, T_C, codes)
        device_fill(KIND_NVFP4_S, seed, T_S8, scales)
        g = NVFP4_GLOBAL_SCALE
    x = torch.empty((M, K), dtype=torch.int16, device=device)
    device_fill(KIND_X, seed, T_X, x)
    return {"fmt": fmt, "M": M, "N": N, "K": K, "codes": codes, "scales": scales, "x": x, "g": g}


# ---------------------------------------------------------------- edge-value problems
#
# Inputs built to reach the corners of the storage formats rather than the
# checkpoint's typical values: negative, subnormal, zero and very large
# scales; groups whose codes are all zero next to ordinary ones; activation
# rows whose magnitudes span many binades.  Drawn from the same counter-based
# generator (tensor ids of their own), so both sides of a parity check get the
# same bits.

T_ADV_CAT = 20     # per (n, group): which scale category
T_ADV_BITS = 21    # per (n, group): random bits of the scale
T_ADV_ZERO = 22    # per (n, group): all-zero-code group
T_ADV_CODE = 23    # per (n, k): codes / weight bytes
T_ADV_XMAG = 24    # per (m, k): activation exponents
T_ADV_X = 25       # per (m, k): activation values

FINITE_E4M3 = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], dtype=np.uint8)


def _adv_u(seed, tensor_id, shape):
    idx = np.arange(int(np.prod(shape)), dtype=np.uint64).reshape(shape)
    return raw64(seed, tensor_id, idx)


def adversarial_problem(fmt: str, seed: int, M: int, N: int, K: int,
                        regime: str = "extreme") -> dict:
    """A problem whose weights and activations sit at the formats' edges.

    regime "extreme": int4 BF16 group scales drawn from six categories per
      (n, group) -- positive and negative normals of moderate size, subnormals
      (either sign), +-0, large (2^60 .. 2^100) and tiny (2^-126 .. 2^-100)
      normals; NVFP4 E4M3 block scales uniform over all 254 finite bytes (sign,
      subnormals and zero included); FP8 weight bytes uniform over the finite
      bytes.  One group in five has all codes equal to zero.  x ~ N(0, 1).
    regime "wide": scales of moderate size (2^-30 .. 2^30, either sign, some
      zero and subnormal), and activation rows whose magnitudes span up to
      2^-24 .. 2^24 within one row: row m % 3 == 0 is N(0, 1), == 1 is
      z * 2^u with u uniform on [-24, 24] per element, == 2 is mostly zero
      with a few large entries.
    The NVFP4 per-tensor scale is fp32(1/448) ("extreme") or 2^-20 ("wide");
    FP8 uses fp32(1/448) or 2^20.
    """
    if regime not in ("extreme", "wide"):
        raise ValueError(regime)
    out = {"fmt": fmt, "M": M, "N": N, "K": K, "regime": regime}
    zero_groups = (_adv_u(seed, T_ADV_ZERO, (N, K // INT4_GROUP)) >> np.uint64(61)) == 0  # 1 in 8
    zero_k = np.repeat(zero_groups, INT4_GROUP, axis=1)
    codes_raw = (_adv_u(seed, T_ADV_CODE, (N, K)) >> np.uint64(56)).astype(np.uint8)
    if fmt == "int4":
        q = ((codes_raw >> 4).astype(np.int16) - 8).astype(np.int8)
        out["codes"] = np.where(zero_k, 0, q).astype(np.int8)
        G = K // INT4_GROUP
        cat = (_adv_u(seed, T_ADV_CAT, (N, G)) % np.uint64(6)).astype(np.int64)
        bits = _adv_u(seed, T_ADV_BITS, (N, G))
        sign = ((bits >> np.uint64(63)) & np.uint64(1)).astype(np.uint16) << 15
        mant = (bits & np.uint64(0x7F)).astype(np.uint16)
        r = ((bits >> np.uint64(8)) % np.uint64(1 << 20)).astype(np.int64)
        if regime == "extreme":
            e_mod = 127 - 8 + r % 12                              # 2^-8 .. 2^3
            e_big = 127 + 60 + r % 41                             # 2^60 .. 2^100
            e_tiny = 1 + r % 27                                   # 2^-126 .. 2^-100
        else:
            e_mod = 127 - 30 + r % 61                             # 2^-30 .. 2^30
            e_big = 127 + r % 31
            e_tiny = 127 - 30 + r % 31
        e = np.select([cat == 0, cat == 1, cat == 2, cat == 3, cat == 4, cat == 5],
                      [e_mod, e_mod, 0, 0, e_big, e_tiny]).astype(np.uint16)
        m = np.where(cat == 3, 0, np.where(cat == 2, np.maximum(mant, 1), mant)).astype(np.uint16)
        s = np.where(cat == 0, 0, sign).astype(np.uint16)         # category 0 positive
        s = np.where(cat == 1, 0x8000, s).astype(np.uint16)        # category 1 negative
        out["scales"] = (s | (e << 7) | m).astype(np.uint16)
        out["g"] = None
    elif fmt == "nvfp4":
        c = codes_raw & np.uint8(0xF)
        zero_code = np.where((codes_raw >> 7) == 1, 8, 0).astype(np.uint8)   # +0 or -0
        out["codes"] = np.where(zero_k, zero_code, c).astype(np.uint8)
        G = K // NVFP4_GROUP
        pick = _adv_u(seed, T_ADV_BITS, (N, G)) % np.uint64(len(FINITE_E4M3))
        sc = FINITE_E4M3[pick.astype(np.int64)]
        out["scales"] = sc.astype(np.uint8)
        out["g"] = float(np.float32(1.0 / 448.0)) if regime == "extreme" else 2.0 ** -20
    elif fmt == "fp8":
        pick = (_adv_u(seed, T_ADV_CODE, (N, K)) >> np.uint64(8)) % np.uint64(len(FINITE_E4M3))
        w8 = FINITE_E4M3[pick.astype(np.int64)]
        out["codes"] = np.where(zero_k, 0, w8).astype(np.uint8)
        out["scales"] = None
        out["g"] = float(np.float32(1.0 / 448.0)) if regime == "extreme" else 2.0 ** 20
    else:
        raise ValueError(fmt)
    # activations
    z = normals(seed, T_ADV_X, np.arange(M * K, dtype=np.uint64).reshape(M, K))
    if regime == "extreme":
        xv = z
    else:
        u = (_adv_u(seed, T_ADV_XMAG, (M, K)) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
        rows = np.arange(M)[:, None] % 3
        wide = z * np.exp2(np.floor(u * 49.0) - 24.0)
        sparse = np.where(u < 0.02, z * 2.0 ** 20, 0.0)
        xv = np.where(rows == 0, z, np.where(rows == 1, wide, sparse))
    out["x"] = to_bf16_bits(xv)
    return out
