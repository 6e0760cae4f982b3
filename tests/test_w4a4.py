"""W4A4 NVFP4 on the GPU against the oracle.

The activation quantiser (g_x, E4M3 block scales, E2M1 codes) must match
oracle.w4a4.quantize_activations bit for bit: every rounding decision is taken
in fp32 on both sides (codes of value zero may differ in sign only).  The
W4A4 matmul must match oracle.w4a4.gemm_w4a4_ref within
|y - y_ref| <= 2^-7 * sum_k |x_hat W| + 1e-3.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import formats
import synth
from bit_weight_only_dequant_b200 import w4a16 as W
from gpu_util import SHAPES, to_device_problem, gscale_tensor, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    W.lib()
    yield


def _x_cases():
    out = []
    for M, K, seed in ((1, 128, 900), (3, 640, 901), (9, 5120, 902), (64, 1024, 903), (16, 17408, 904)):
        out.append((f"normal M={M} K={K}", synth.activations(seed, M, K)))
    # rows spanning many binades, mostly-zero rows and all-zero blocks
    wide = synth.adversarial_problem("int4", 905, 6, 1, 2048, "wide")["x"].copy()
    wide[0, 32:48] = 0
    out.append(("wide", wide))
    z = np.zeros((2, 256), np.uint16)
    out.append(("all zero", z))
    # values on the grid: each block reaches the top code exactly
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 16, size=(4, 256)).astype(np.uint8)
    codes[:, ::16] = 7
    s8 = rng.integers(0x18, 0x70, size=(4, 16)).astype(np.uint8)
    x = formats.e2m1_to_f64(codes) * np.repeat(formats.e4m3_to_f64(s8), 16, axis=1) * 2.0 ** -7
    out.append(("representable", formats.f64_to_bf16_rne(x)))
    return out


@pytest.mark.parametrize("case", range(len(_x_cases())))
def test_activation_quantiser_bit_exact(case):
    t = torch()
    name, x_bits = _x_cases()[case]
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    codes, scales, g_x = W.quantize_act_nvfp4(x)
    t.cuda.synchronize()
    g_ref = oracle.w4a4.activation_global_scale(x_bits)
    q_ref, s_ref = oracle.w4a4.quantize_activations(x_bits, g_ref)
    g = g_x.cpu().numpy()[0]
    assert np.float32(g).view(np.uint32) == np.float32(g_ref).view(np.uint32), (name, g, g_ref)
    s = scales.cpu().numpy()
    assert np.array_equal(s, s_ref), (name, np.argwhere(s != s_ref)[:5])
    q = codes.cpu().numpy()
    same = (q == q_ref) | (((q & 7) == 0) & ((q_ref & 7) == 0))      # +-0 may differ in sign only
    assert same.all(), (name, np.argwhere(~same)[:5])
    assert np.all(q <= 15)


def _gemm_case(M, N, K, seed, path):
    t = torch()
    x_bits = synth.activations(seed, M, K)
    pw_ = synth.problem("nvfp4", seed + 1, 1, N, K)
    codes, scales, _ = to_device_problem(pw_)
    pw, ps = W.pack_on_device("nvfp4", N, K, codes, scales)
    g_w = gscale_tensor(pw_["g"])
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    y = W.gemm_w4a4(x, pw, ps, N, g_w, path=path)
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    return x_bits, pw_, y.float().cpu().numpy().astype(np.float64)


def _assert_w4a4_parity(y, x_bits, pw_, cols=None, what=""):
    g_x = oracle.w4a4.activation_global_scale(x_bits)
    xq, xs = oracle.w4a4.quantize_activations(x_bits, g_x)
    wc, wsc = pw_["codes"], pw_["scales"]
    y_ref = oracle.w4a4.gemm_w4a4_ref(xq, xs, g_x, wc, wsc, pw_["g"])
    xh = oracle.w4a4.dequant_activations(xq, xs, g_x)
    wh = oracle.w4a4.weights_exact(wc, wsc, pw_["g"])
    bound = np.abs(xh) @ np.abs(wh).T
    if cols is not None:
        y = y[:, cols]
    allowed = oracle.TOL_REL * bound + oracle.TOL_ABS
    err = np.abs(y - y_ref)
    assert np.all(err <= allowed), (what, int((err > allowed).sum()), float((err / allowed).max()))


@pytest.mark.parametrize("M,N,K,path", [(1, 256, 512, W.PATH_AUTO), (3, 1000, 1024, W.PATH_GEMV),
                                        (9, 304, 1152, W.PATH_TC), (16, 160, 3072, W.PATH_GEMV),
                                        (64, 272, 640, W.PATH_TC), (200, 96, 384, W.PATH_TC),
                                        (2, 24, 17408, W.PATH_GEMV), (1, 1, 128, W.PATH_AUTO)])
def test_w4a4_gemm_parity_small(M, N, K, path):
    x_bits, pw_, y = _gemm_case(M, N, K, 950 + M, path)
    _assert_w4a4_parity(y, x_bits, pw_, what=f"W4A4 M={M} N={N} K={K} path={path}")


@pytest.mark.parametrize("name,M", [(n, M) for n in ("qkv", "o", "gate_up", "down") for M in (1, 9, 64)])
def test_w4a4_gemm_parity_full_shapes_sampled(name, M):
    t = torch()
    K, N = SHAPES[name]
    seed = 960
    x_bits = synth.activations(seed, M, K)
    p = synth.device_problem("nvfp4", seed + 1, 1, N, K)
    pw, ps = W.pack_on_device("nvfp4", N, K, p["codes"], p["scales"])
    del p
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    y = W.gemm_w4a4(x, pw, ps, N, gscale_tensor(synth.NVFP4_GLOBAL_SCALE))
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    rows = np.unique(np.concatenate([[0, 15, 16, N - 1], np.random.default_rng(M).integers(0, N, 40)]))
    ph = synth.problem("nvfp4", seed + 1, 1, N, K, rows=rows)
    _assert_w4a4_parity(y.float().cpu().numpy().astype(np.float64), x_bits, ph, cols=rows,
                        what=f"W4A4 {name} M={M}")
    del pw, ps, y
    t.cuda.empty_cache()


def test_w4a4_rejects_bad_arguments():
    t = torch()
    x = t.zeros((2, 256), dtype=t.bfloat16, device="cuda")
    assert W.w4a16_gemm_w4a4(2, 16, 200, x, 1 << 20, 1 << 20, 1 << 20, 1 << 20) == W.ERR_SHAPE
    assert W.w4a16_gemm_w4a4(2, 16, 256, x, 1 << 20, 1 << 20, None, 1 << 20) == W.ERR_ARG
    assert W.w4a16_quantize_act_nvfp4(2, 250, x, 1 << 20, 1 << 20, 1 << 20) == W.ERR_SHAPE


# ---------------------------------------------------------------- block-scaled tensor-core path

def _bs_weights(seed, N, K):
    pw_ = synth.problem("nvfp4", seed, 1, N, K)
    codes, scales, _ = to_device_problem(pw_)
    pw, psf = W.pack_on_device("nvfp4_bs", N, K, codes, scales)
    return pw_, pw, psf


def test_block_scaled_device_packer_matches_host_packer():
    N, K = 300, 384
    pw_, pw, psf = _bs_weights(980, N, K)
    w = np.zeros(W.w4a16_packed_weight_bytes(W.FMT_NVFP4_BS, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(W.FMT_NVFP4_BS, N, K), np.uint8)
    assert W.w4a16_pack_host(W.FMT_NVFP4_BS, N, K, pw_["codes"], pw_["scales"], w, s) == W.OK
    assert np.array_equal(pw.cpu().numpy(), w)
    assert np.array_equal(psf.cpu().numpy(), s)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (3, 1000, 1024), (9, 304, 1152), (16, 160, 3072),
                                   (64, 272, 640), (200, 96, 384), (2, 24, 17408), (1, 1, 128),
                                   (130, 130, 256), (64, 129, 384), (128, 512, 2048),
                                   (1000, 200, 512)])
def test_w4a4_block_scaled_parity_small(M, N, K):
    t = torch()
    x_bits = synth.activations(970 + M, M, K)
    pw_, pw, psf = _bs_weights(971 + M, N, K)
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    y = W.gemm_w4a4_bs(x, pw, psf, N, gscale_tensor(pw_["g"]))
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    _assert_w4a4_parity(y.float().cpu().numpy().astype(np.float64), x_bits, pw_,
                        what=f"W4A4 block-scaled M={M} N={N} K={K}")


def test_w4a4_block_scaled_parity_wide_activations():
    # rows spanning many binades: block scales far below the tensor's largest
    # (E4M3 subnormals and zeros), all-zero blocks, sparse large elements
    t = torch()
    M, N, K = 12, 200, 2048
    x_bits = synth.adversarial_problem("int4", 985, M, 1, K, "wide")["x"].copy()
    x_bits[1, 64:96] = 0
    pw_, pw, psf = _bs_weights(986, N, K)
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    y = W.gemm_w4a4_bs(x, pw, psf, N, gscale_tensor(pw_["g"]))
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    _assert_w4a4_parity(y.float().cpu().numpy().astype(np.float64), x_bits, pw_, what="wide rows")


@pytest.mark.parametrize("name,M", [(n, M) for n in ("qkv", "o", "gate_up", "down") for M in (1, 9, 64)])
def test_w4a4_block_scaled_full_shapes_sampled(name, M):
    t = torch()
    K, N = SHAPES[name]
    seed = 990
    x_bits = synth.activations(seed, M, K)
    p = synth.device_problem("nvfp4", seed + 1, 1, N, K)
    pw, psf = W.pack_on_device("nvfp4_bs", N, K, p["codes"], p["scales"])
    del p
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    y = W.gemm_w4a4_bs(x, pw, psf, N, gscale_tensor(synth.NVFP4_GLOBAL_SCALE))
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], np.random.default_rng(M).integers(0, N, 40)]))
    ph = synth.problem("nvfp4", seed + 1, 1, N, K, rows=rows)
    _assert_w4a4_parity(y.float().cpu().numpy().astype(np.float64), x_bits, ph, cols=rows,
                        what=f"W4A4 block-scaled {name} M={M}")
    del pw, psf, y
    t.cuda.empty_cache()


def test_w4a4_block_scaled_rejects_bad_arguments():
    t = torch()
    x = t.zeros((2, 256), dtype=t.bfloat16, device="cuda")
    assert W.w4a16_gemm_w4a4_bs(2, 16, 200, x, 1 << 20, 1 << 20, 1 << 20, 1 << 20) == W.ERR_SHAPE
    assert W.w4a16_gemm_w4a4_bs(0, 16, 256, x, 1 << 20, 1 << 20, 1 << 20, 1 << 20) == W.ERR_SHAPE
    assert W.w4a16_gemm_w4a4_bs(2, 16, 256, x, 1 << 20, 1 << 20, None, 1 << 20) == W.ERR_ARG
    assert W.w4a16_gemm_w4a4_bs(2, 16, 256, x, (1 << 20) + 8, 1 << 20, 1 << 20, 1 << 20) == W.ERR_ALIGN


def test_w4a4_block_scaled_reads_weights_packed_just_before():
    # the block-scaled matmul loads its weights before its dependent-launch
    # wait; weights packed by the kernel right before the call (same stream,
    # no host synchronisation) must still be read complete
    t = torch()
    M, N, K = 4, 1024, 4096
    x_bits = synth.activations(995, M, K)
    pw_ = synth.problem("nvfp4", 996, 1, N, K)
    codes, scales, _ = to_device_problem(pw_)
    x = t.from_numpy(np.ascontiguousarray(x_bits.view(np.int16))).cuda().view(t.bfloat16)
    g_w = gscale_tensor(pw_["g"])
    s = t.cuda.Stream()
    t.cuda.synchronize()
    with t.cuda.stream(s):
        for _ in range(3):
            pw, psf = W.pack_on_device("nvfp4_bs", N, K, codes, scales, stream=s)
            y = W.gemm_w4a4_bs(x, pw, psf, N, g_w, stream=s)
    s.synchronize()
    W.check(W.w4a16_device_status(s), "device status")
    _assert_w4a4_parity(y.float().cpu().numpy().astype(np.float64), x_bits, pw_,
                        what="weights packed just before")
