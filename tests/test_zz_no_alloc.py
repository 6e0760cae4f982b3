"""w4a16_gemm_noalloc: the GEMV entry point that allocates no device memory.

Callers that cannot allocate (an application that owns all device memory
through its own pool, or a steady state that must not call cudaMalloc because
an allocation can synchronise the device) use this entry point instead of
w4a16_gemm; its split-K scratch is a fixed array inside the library.  Its
results must match those of w4a16_gemm, and the oracle within the accuracy
contract, call after call, although every call reuses the same scratch.

Collected last on purpose (file name), and self-contained so that it passes
alone in a fresh process as well as after the rest of the suite.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from bit_weight_only_dequant_b200 import w4a16 as W

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _weights(p):
    if p["fmt"] == "int4":
        return oracle.dequant_int4_g128(p["codes"], p["scales"])
    if p["fmt"] == "fp8":
        return oracle.dequant_fp8_e4m3(p["codes"], p["g"])
    return oracle.dequant_nvfp4(p["codes"], p["scales"], p["g"])


@pytest.mark.parametrize("fmt,M,N,K,seed", [
    ("int4", 8, 5120, 17408, 4),   # the down projection: split-K, uses the scratch
    ("int4", 1, 17408, 5120, 3),
    ("nvfp4", 3, 1000, 1024, 51),
    ("int4", 16, 400, 3072, 90),
    ("fp8", 4, 1000, 2048, 91),
    ("fp8", 2, 512, 17408, 92),    # FP8 with a long K: split-K through the scratch
])
def test_noalloc_matches_gemm_on_consecutive_calls(fmt, M, N, K, seed):
    t = _torch()
    f = W.FMTS[fmt]
    p = synth.device_problem(fmt, seed, M, N, K)
    pw, ps = W.pack_on_device(fmt, N, K, p["codes"], p["scales"])
    g = None if p["g"] is None else t.tensor([p["g"]], dtype=t.float32, device="cuda")
    x = p["x"].view(t.bfloat16)
    y_ref = t.empty((M, N), dtype=t.bfloat16, device="cuda")
    W.check(W.w4a16_gemm(f, M, N, K, x, pw, ps, g, y_ref), "w4a16_gemm")
    ys = [t.full((M, N), float("nan"), dtype=t.bfloat16, device="cuda") for _ in range(3)]
    # first call: per-device set-up, then two more calls in a row on the same scratch
    W.check(W.w4a16_gemm_noalloc(f, M, N, K, x, pw, ps, g, ys[0]), "first call")
    t.cuda.synchronize()
    free_before = t.cuda.mem_get_info()[0]
    for y in ys[1:]:
        W.check(W.w4a16_gemm_noalloc(f, M, N, K, x, pw, ps, g, y), "w4a16_gemm_noalloc")
    t.cuda.synchronize()
    assert t.cuda.mem_get_info()[0] == free_before, "a call allocated device memory"

    ref = y_ref.float().cpu().numpy().astype(np.float64)
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(seed).integers(0, N, 64)]))
    ph = synth.problem(fmt, seed, M, N, K, rows=rows)
    w = _weights(ph)
    y_oracle = oracle.gemm_ref(ph["x"], w)
    bound = oracle.abs_bound(ph["x"], w)
    allowed = oracle.TOL_REL * bound + oracle.TOL_ABS
    for y in ys:
        got = y.float().cpu().numpy().astype(np.float64)
        assert not np.isnan(got).any()
        # against the oracle on the sampled columns, and against w4a16_gemm
        assert np.all(np.abs(got[:, rows] - y_oracle) <= allowed)
        assert np.all(np.abs(got[:, rows] - ref[:, rows]) <= allowed)
        if W.w4a16_gemm_path(f, M, N, K) == W.PATH_GEMV:
            # same kernel and same reduction order as w4a16_gemm on this path
            assert np.array_equal(got, ref)


def test_noalloc_rejects_what_does_not_fit():
    _torch()
    fake = 1 << 20  # aligned, never dereferenced: the call returns before any launch
    # split-K partials of a 248,320-column output at M = 16 far exceed the
    # scratch.  Checked on the host first: if the planner ever chose no K split
    # here, the call would need no scratch and would launch on the fake
    # pointers, so the test stops before making it.
    M, N, K = 16, 248320, 17408
    path, plan = W.w4a16_plan(W.PATH_GEMV, 0, M, N, K, 0, 148)
    assert path == W.PATH_GEMV and plan[0] > 1, plan
    import torch
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    path, plan = W.w4a16_plan(W.PATH_GEMV, 0, M, N, K, 0, props.multi_processor_count)
    assert path == W.PATH_GEMV and plan[0] > 1, plan
    assert plan[0] * M * ((N + 15) // 16 * 16) * 4 > (8 << 20)
    assert W.w4a16_gemm_noalloc(0, M, N, K, fake, fake, fake, None, fake) == W.ERR_SCRATCH
    assert W.w4a16_gemm_noalloc(0, 17, 256, 512, fake, fake, fake, None, fake) == W.ERR_SHAPE
    assert W.w4a16_gemm_noalloc(0, 1, 256, 500, fake, fake, fake, None, fake) == W.ERR_SHAPE
    assert W.w4a16_gemm_noalloc(1, 1, 256, 512, fake, fake, fake, None, fake) == W.ERR_ARG
    assert W.status_string(W.ERR_SCRATCH).startswith("W4A16_ERR_SCRATCH")
