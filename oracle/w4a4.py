"""W4A4 NVFP4: the activations quantised to NVFP4 as well (fp64, numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Groundwork for a
block-scaled tensor-core path that is not built yet.

The pages name the format only: compressed-tensors "W4A4 NVFP4" with group
size 16 (model card "SuperQwen3.8-27b-abliterated-NVFP4-2xDGX", table "Release
highlights").  Reading, the plainest one consistent with the weight side of
the same format:
* one fp32 activation scale per tensor, g_x = amax|x| / (6 * 448), formed in
  fp32 from the tensor itself (calibration on the data at hand);
* one E4M3 scale per (row m, 16-group j): s = RNE_e4m3(amax_block / (6 g_x)),
  the division and the product 6 g_x in fp32, saturating at 448;
* codes q = RNE_e2m1(x / (e4m3(s) * g_x)), the product and the division in
  fp32, saturating at +-6 (a zero scale gives zero codes);
* x_hat = e2m1(q) * e4m3(s) * g_x, and y = sum_k W[n][k] * x_hat[m][k] with the
  weights' own exact values e2m1 * e4m3 * g_w (no BF16 rounding on either
  side: a block-scaled MMA multiplies the 4-bit values and applies the scales).
The fp32 steps fix every rounding decision, so a kernel can take the same
decisions in the same precision.
"""

from __future__ import annotations

import numpy as np

from .formats import bf16_to_f64, e2m1_to_f64, e4m3_to_f64, f64_to_e2m1_rne, f64_to_e4m3_rne

GROUP = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def activation_global_scale(x_bits: np.ndarray) -> float:
    """g_x = fp32(amax|x|) / fp32(6 * 448), an fp32 value (1.0 for an all-zero x)."""
    amax = np.float32(np.max(np.abs(bf16_to_f64(x_bits)), initial=0.0))
    if amax == 0:
        return 1.0
    return float(amax / np.float32(E2M1_MAX * E4M3_MAX))


def quantize_activations(x_bits: np.ndarray, g_x: float):
    """BF16 x [M][K] -> (e2m1 codes [M][K] uint8, E4M3 scales [M][K/16] uint8)."""
    x = bf16_to_f64(x_bits).astype(np.float32)                # exact: BF16 is a binary32 subset
    M, K = x.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 16")
    g = np.float32(g_x)
    blocks = x.reshape(M, K // GROUP, GROUP)
    amax = np.max(np.abs(blocks), axis=2)                      # exact in fp32
    t = amax / (np.float32(E2M1_MAX) * g)                      # fp32 product, fp32 division
    s8 = f64_to_e4m3_rne(t.astype(np.float64))
    step = (e4m3_to_f64(s8).astype(np.float32) * g)           # fp32 product
    with np.errstate(divide="ignore", invalid="ignore"):
        v = blocks / step[:, :, None]                          # fp32 division
    v = np.where(step[:, :, None] > 0, v, np.float32(0.0))
    codes = f64_to_e2m1_rne(v.astype(np.float64)).reshape(M, K)
    return codes, s8


def dequant_activations(codes: np.ndarray, s8: np.ndarray, g_x: float) -> np.ndarray:
    """x_hat[m][k] = e2m1(q) * e4m3(s[m][k // 16]) * g_x, exact in fp64."""
    return e2m1_to_f64(codes) * np.repeat(e4m3_to_f64(s8), GROUP, axis=1) * float(np.float32(g_x))


def weights_exact(codes: np.ndarray, s8: np.ndarray, g_w: float) -> np.ndarray:
    """The NVFP4 weights' exact values e2m1 * e4m3 * g_w (no rounding), fp64 [N][K]."""
    return e2m1_to_f64(codes) * np.repeat(e4m3_to_f64(s8), GROUP, axis=1) * float(np.float32(g_w))


def gemm_w4a4_ref(x_codes, x_s8, g_x, w_codes, w_s8, g_w) -> np.ndarray:
    """y[m][n] = sum_k x_hat[m][k] * W[n][k] in fp64.

    The block-scaled parts e2m1 * e4m3 have at most 6 significant bits on each
    side, so their products and the sum over k are exact in binary64 for K up
    to about 2^10 (and within 2^-53 relative beyond); the two per-tensor fp32
    scales multiply the sum at the end (two roundings of 2^-53).
    """
    a = e2m1_to_f64(x_codes) * np.repeat(e4m3_to_f64(x_s8), GROUP, axis=1)
    b = e2m1_to_f64(w_codes) * np.repeat(e4m3_to_f64(w_s8), GROUP, axis=1)
    return (a @ b.T) * float(np.float32(g_x)) * float(np.float32(g_w))
