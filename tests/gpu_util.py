"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs.  The CUDA side is reached only through the C ABI binding."""

from __future__ import annotations

import numpy as np

import oracle
import synth
from bit_weight_only_dequant_b200 import w4a16 as W

# The linear shapes of the 5120-hidden, 64-layer dense model (K -> N).
SHAPES = {
    "qkv": (5120, 8192),      # fused Q (24 x 256) + K, V (2 x 4 x 256)
    "o": (6144, 5120),
    "gate_up": (5120, 34816),  # fused gate and up, intermediate 17408
    "down": (17408, 5120),
    "target": (5120, 17408),  # one half of gate/up: the M = 1 bandwidth target
}
SEEDS = {"qkv": 1, "o": 2, "gate_up": 3, "down": 4, "target": 3}


def torch():
    import torch as _t
    return _t


def to_device_problem(p):
    """Host numpy problem -> torch CUDA tensors (same bits)."""
    t = torch()
    codes = t.from_numpy(np.ascontiguousarray(p["codes"])).cuda()
    sc = p["scales"]
    scales = None if sc is None else t.from_numpy(
        np.ascontiguousarray(sc.view(np.int16) if sc.dtype == np.uint16 else sc)).cuda()
    x = t.from_numpy(np.ascontiguousarray(p["x"].view(np.int16))).cuda()
    return codes, scales, x


def gscale_tensor(g):
    t = torch()
    if g is None:
        return None
    return t.tensor([g], dtype=t.float32, device="cuda")


def run_gemm(fmt, codes, scales, x, N, g=None, path=W.PATH_AUTO, y=None):
    """Pack on device and run the GEMM; returns (y as float64 numpy, packed)."""
    t = torch()
    M, K = x.shape
    pw, ps = W.pack_on_device(fmt, N, K, codes, scales)
    gt = gscale_tensor(g)
    xb = x.view(t.bfloat16)
    out = W.gemm(fmt, xb, pw, ps, N, global_scale=gt, y=y, path=path)
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    return out.float().cpu().numpy().astype(np.float64), (pw, ps, gt)


def oracle_weights(p):
    if p["fmt"] == "int4":
        return oracle.dequant_int4_g128(p["codes"], p["scales"])
    if p["fmt"] == "fp8":
        return oracle.dequant_fp8_e4m3(p["codes"], p["g"])
    return oracle.dequant_nvfp4(p["codes"], p["scales"], p["g"])


def assert_parity(y_gpu, x_bits, w_bits, what=""):
    y_ref = oracle.gemm_ref(x_bits, w_bits)
    bound = oracle.abs_bound(x_bits, w_bits)
    ok, excess = oracle.within_tolerance(y_gpu, y_ref, bound)
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        detail = [(int(m), int(n), float(y_gpu[m, n]), float(y_ref[m, n]), float(bound[m, n]))
                  for m, n in bad]
        raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance, e.g. {detail}")
    return float(excess.max())


def bf16_bits(t_bf16):
    t = torch()
    return t_bf16.view(t.int16).cpu().numpy().view(np.uint16)
