"""Dequantise-then-matmul in fp64: the definition the CUDA path must match.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The method (the decode-time weight-only 4-bit linear of the 5120-hidden dense
model) is fixed by two checkpoint contracts on the pages:

* INT4, forum post "Qwen3.8-27B on single DGX Spark ...", section "Quality":
  symmetric GPTQ, 4-bit, one scale per group of 128 K-elements, no zero point,
  no act-order, BF16 activations.  Reading: q is an integer in [-8, 7], the
  scale is a BF16 value per (output column n, K-group), and the dequantised
  weight is the BF16 value nearest to q * s.
* NVFP4, model card "Qwen3.8 27B - NVFP4 for veloGB10", section
  "Specifications" (compressed-tensors nvfp4-pack-quantized), group size 16 per
  the "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX" card; W4A16 use on Blackwell
  per "Qwen3.8-27B on DGX Spark (GB10): vLLM 0.24 + NVFP4 ...", section "What
  Spark-native means".  Reading: the weight is an E2M1 value times an E4M3
  scale per (n, 16-group) times one fp32 scale per tensor, rounded once to
  BF16; the activations stay BF16.

The pages' bandwidth argument (blog post "One Config Line Made My 27B Model
2.7x Faster", section "Gotcha #2") is what makes this the hot path: decode
speed is set by the bytes of weights streamed per token.

Accuracy contract: per element |y - y_ref| <= 2**-7 * sum_k |W_deq[n][k] *
x[m][k]| + 1e-3, and exported dequantised weights bit-exact.

Fused gate/up projection (the MLP of every layer, named on the pages only as
"MLP" linears: model card "Qwen3.8 27B - NVFP4 for veloGB10", section
"Specifications"; guide "Qwen3.8-27B on DGX Spark (GB10)", section "What
Spark-native means").  Reading, the plainest one for this model family: the
packed [2I][K] weight holds the gate rows first and the up rows second, and
the layer's output is h = SiLU(gate) * up with SiLU(z) = z / (1 + e^-z).
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64, e2m1_to_f64, e4m3_to_f64, f64_to_bf16_rne

INT4_GROUP = 128
NVFP4_GROUP = 16
TOL_REL = 2.0 ** -7
TOL_ABS = 1e-3


def dequant_int4_g128(q: np.ndarray, scale_bits: np.ndarray) -> np.ndarray:
    """W_deq[n][k] = RNE_bf16(q[n][k] * s[n][k // 128]); returns BF16 bits [N][K].

    q: int8 [N][K] in [-8, 7].  scale_bits: uint16 BF16 patterns [N][K/128].
    The product of a 4-bit integer and an 8-significant-bit BF16 value is exact
    in binary64, so the only rounding is the one onto BF16.
    """
    q = np.asarray(q)
    N, K = q.shape
    if K % INT4_GROUP:
        raise ValueError("K must be a multiple of the group size 128")
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("int4 values must lie in [-8, 7]")
    s = bf16_to_f64(scale_bits)
    if s.shape != (N, K // INT4_GROUP):
        raise ValueError("scale shape must be [N][K/128]")
    s_per_k = np.repeat(s, INT4_GROUP, axis=1)           # s[n][k // 128]
    return f64_to_bf16_rne(q.astype(np.float64) * s_per_k)


def dequant_nvfp4(codes: np.ndarray, scale_e4m3: np.ndarray, g: float) -> np.ndarray:
    """W_deq[n][k] = RNE_bf16(e2m1(c[n][k]) * e4m3(s8[n][k // 16]) * g); BF16 bits.

    codes: uint8 [N][K] in 0..15.  scale_e4m3: uint8 [N][K/16] (finite).
    g: the fp32 per-tensor scale (a Python float holding an fp32 value).
    e2m1 (2 significant bits) * e4m3 (4) * fp32 (24) has at most 30 significant
    bits, exact in binary64, so the product is rounded once onto BF16.
    """
    c = np.asarray(codes)
    N, K = c.shape
    if K % NVFP4_GROUP:
        raise ValueError("K must be a multiple of the group size 16")
    if c.max(initial=0) > 15:
        raise ValueError("e2m1 codes must lie in 0..15")
    s = e4m3_to_f64(scale_e4m3)
    if s.shape != (N, K // NVFP4_GROUP):
        raise ValueError("scale shape must be [N][K/16]")
    if not np.all(np.isfinite(s)):
        raise ValueError("NaN E4M3 scales are not allowed")
    g64 = float(np.float32(g))
    s_per_k = np.repeat(s, NVFP4_GROUP, axis=1)
    return f64_to_bf16_rne(e2m1_to_f64(c) * s_per_k * g64)


def dequant_fp8_e4m3(codes: np.ndarray, g: float) -> np.ndarray:
    """W_deq[n][k] = RNE_bf16(e4m3(w8[n][k]) * g); BF16 bits [N][K].

    FP8 weight-only variant (W8A16) of the attention linears, which the NVFP4
    checkpoint keeps in FP8 (guide "Qwen3.8-27B on DGX Spark (GB10)", section
    "The right stack for Spark").  Reading: E4M3 bytes with one fp32 scale per
    tensor.  e4m3 (4 significant bits) * fp32 (24) is exact in binary64, so the
    product is rounded once onto BF16.  w8: uint8 [N][K] (NaN bytes rejected).
    """
    c = np.asarray(codes, dtype=np.uint8)
    v = e4m3_to_f64(c)
    if not np.all(np.isfinite(v)):
        raise ValueError("NaN E4M3 weights are not allowed")
    g64 = float(np.float32(g))
    return f64_to_bf16_rne(v * g64)


def gemm_ref(x_bits: np.ndarray, w_bits: np.ndarray) -> np.ndarray:
    """y_ref[m][n] = sum_k x[m][k] * W_deq[n][k] in binary64 (unrounded).

    x_bits: BF16 [M][K]; w_bits: BF16 [N][K].  Returns float64 [M][N].
    """
    x = bf16_to_f64(x_bits)
    w = bf16_to_f64(w_bits)
    return x @ w.T


def abs_bound(x_bits: np.ndarray, w_bits: np.ndarray) -> np.ndarray:
    """sum_k |W_deq[n][k] * x[m][k]| as float64 [M][N] (scale of the tolerance)."""
    return np.abs(bf16_to_f64(x_bits)) @ np.abs(bf16_to_f64(w_bits)).T


def within_tolerance(y: np.ndarray, y_ref: np.ndarray, bound: np.ndarray):
    """Elementwise check of the accuracy contract; returns (ok_mask, excess).

    ``excess`` is |y - y_ref| divided by the allowed error (<= 1 passes).
    """
    allowed = TOL_REL * bound + TOL_ABS
    err = np.abs(np.asarray(y, dtype=np.float64) - y_ref)
    return err <= allowed, err / allowed


# ---------------------------------------------------------------- fused gate/up + SiLU

SILU_LIPSCHITZ = 1.1   # max over z of |d/dz (z * sigmoid(z))| is 1.0998...


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z)), binary64, elementwise.

    exp(-z) overflows to +inf for z < -709; z / inf is then -0.0, the limit.
    """
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gate_up_silu_ref(x_bits: np.ndarray, w_bits: np.ndarray):
    """h[m][i] = SiLU(gate[m][i]) * up[m][i] in binary64 (unrounded).

    w_bits: BF16 [2I][K], gate rows [0, I), up rows [I, 2I).  gate and up are
    the exact products of gemm_ref.  Returns (h, gate, up), float64 [M][I].
    """
    N = w_bits.shape[0]
    if N % 2:
        raise ValueError("the fused gate/up weight has an even number of rows")
    I = N // 2
    y = gemm_ref(x_bits, w_bits)
    gate, up = y[:, :I], y[:, I:]
    return silu(gate) * up, gate, up


def gate_up_silu_allowed(x_bits: np.ndarray, w_bits: np.ndarray, gate: np.ndarray,
                         up: np.ndarray) -> np.ndarray:
    """Allowed |h - h_ref| per element for the fused output.

    Each of gate and up may carry the matmul's own error e = 2^-7 * sum_k
    |W_deq x| + 1e-3.  SiLU is 1.1-Lipschitz, so |SiLU(g') u' - SiLU(g) u| <=
    (|SiLU(g)| + 1.1 e_g) e_u + 1.1 e_g |u|; the BF16 rounding of the output
    and the fp32 evaluation of SiLU add at most 2^-7 |h| (RNE onto BF16 alone
    is 2^-8 relative), and 1e-3 absolute covers the rest.
    """
    N = w_bits.shape[0]
    I = N // 2
    b = abs_bound(x_bits, w_bits)
    e_g = TOL_REL * b[:, :I] + TOL_ABS
    e_u = TOL_REL * b[:, I:] + TOL_ABS
    sg = silu(gate)
    h = sg * up
    return ((np.abs(sg) + SILU_LIPSCHITZ * e_g) * e_u + SILU_LIPSCHITZ * e_g * np.abs(up)
            + TOL_REL * np.abs(h) + TOL_ABS)
