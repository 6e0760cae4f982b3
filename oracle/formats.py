"""Storage-type decoders and BF16 rounding for the oracle (fp64, numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources of the formats:
* BF16 activations and BF16 group scales: the INT4 checkpoint contract in the
  NVIDIA developer-forum post "Qwen3.8-27B on single DGX Spark ..." (section
  "Quality": symmetric GPTQ, 4-bit, group 128, BF16 activations, no act-order,
  no zero points).
* FP4 (E2M1) values and FP8-E4M3 group scales: the NVFP4 checkpoint format of
  the model card "Qwen3.8 27B - NVFP4 for veloGB10" (section "Specifications",
  compressed-tensors nvfp4-pack-quantized) and the group size 16 of the
  "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX" card (section "Release
  highlights").  The pages do not spell out the bit layouts; the decoders follow
  the OCP Microscaling (MX) v1.0 definitions of E2M1 and E4M3 (E4M3: bias 7, no
  infinities, S.1111.111 is NaN, largest finite 448; E2M1: bias 1, one mantissa
  bit, largest 6).
"""

from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) -> float64.  BF16 is the top half of a binary32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(b: np.ndarray) -> np.ndarray:
    """OCP FP8-E4M3 bytes -> float64 (NaN for S.1111.111)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    exp = (b >> 3) & 0xF
    man = b & 0x7
    normal = np.ldexp(1.0 + man / 8.0, exp - 7)
    subnormal = np.ldexp(man / 8.0, -6)
    v = sign * np.where(exp == 0, subnormal, normal)
    return np.where((exp == 0xF) & (man == 0x7), np.nan, v)


def e2m1_to_f64(c: np.ndarray) -> np.ndarray:
    """FP4-E2M1 codes (low 4 bits used) -> float64.

    Bit 3 is the sign, bits 2..1 the exponent (bias 1), bit 0 the mantissa;
    exponent 0 is subnormal (value = mantissa * 0.5).
    """
    c = np.asarray(c, dtype=np.uint8).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    exp = (c >> 1) & 0x3
    man = c & 0x1
    v = np.where(exp == 0, man * 0.5, np.ldexp(1.0 + man / 2.0, exp - 1))
    return sign * v


def f64_to_bf16_rne(v: np.ndarray) -> np.ndarray:
    """Round exact float64 values to BF16, round-to-nearest ties-to-even.

    Returns uint16 bit patterns.  The argument must hold the exact value to be
    rounded (the callers form products that binary64 represents exactly), so
    this is the single rounding of the exact product.  Subnormal BF16 results
    (magnitude below 2**-126, quantum 2**-133) are kept; overflow gives +-inf;
    zero keeps its sign.
    """
    v = np.asarray(v, dtype=np.float64)
    mant, ex = np.frexp(v)                         # v = mant * 2**ex, 0.5 <= |mant| < 1
    # 8 significant bits in the normal range; np.rint rounds half to even.
    r = np.ldexp(np.rint(np.ldexp(mant, 8)), ex - 8)
    tiny = np.abs(v) < 2.0 ** -126
    r = np.where(tiny, np.ldexp(np.rint(np.ldexp(v, 133)), -133), r)
    big = np.abs(r) > float(np.finfo(np.float32).max)
    with np.errstate(over="ignore"):
        r32 = np.where(big, np.copysign(np.inf, v), r).astype(np.float32)
    bits = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    # keep the sign of zero results (rint(-tiny) is -0.0 already; be explicit)
    zero = r == 0
    bits = np.where(zero, np.where(np.signbit(v), np.uint16(0x8000), np.uint16(0)), bits)
    return bits.astype(np.uint16)


def f64_to_e4m3_rne(v: np.ndarray) -> np.ndarray:
    """Round non-negative float64 values to OCP FP8-E4M3 bytes, nearest, ties to even.

    Saturates at 448 (0x7E), the largest finite value; never produces the NaN
    pattern.  Normal range: 4 significant bits; subnormals (below 2**-6):
    quantum 2**-9.  Used for block scales, which are non-negative.
    """
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("E4M3 block scales are rounded from non-negative values")
    m, e = np.frexp(v)
    r = np.ldexp(np.rint(np.ldexp(m, 4)), e - 4)
    r = np.where(v < 2.0 ** -6, np.ldexp(np.rint(np.ldexp(v, 9)), -9), r)
    r = np.minimum(r, 448.0)
    out = np.zeros(v.shape, dtype=np.uint8)
    sub = (r > 0) & (r < 2.0 ** -6)
    out[sub] = np.ldexp(r[sub], 9).astype(np.uint8)
    nrm = r >= 2.0 ** -6
    mm, ee = np.frexp(r[nrm])
    out[nrm] = (((ee - 1 + 7).astype(np.int64) << 3) | (np.ldexp(mm, 4) - 8).astype(np.int64)).astype(np.uint8)
    return out


E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def f64_to_e2m1_rne(v: np.ndarray) -> np.ndarray:
    """Round float64 values to FP4-E2M1 codes, nearest, ties to the even code.

    Magnitudes at or above 6 saturate to 6 (code 7); the sign goes to bit 3
    (negative zero included).  "Even" is the code whose mantissa bit is 0.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    grid = np.array(E2M1_MAGNITUDES)
    lo = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    mag = np.where(a >= 6.0, 7, np.where(pick_hi, hi, lo))
    return (mag | np.where(np.signbit(v), 8, 0)).astype(np.uint8)
