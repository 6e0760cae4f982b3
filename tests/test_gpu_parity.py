"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Bars: dequantised weights bit-exact; GEMM outputs within
|y - y_ref| <= 2^-7 * sum_k |W_deq x| + 1e-3 per element.
"""

from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from oracle import formats
import synth
from bit_weight_only_dequant_b200 import w4a16 as W
from gpu_util import (SEEDS, SHAPES, assert_parity, bf16_bits, gscale_tensor, oracle_weights,
                      run_gemm, to_device_problem, torch)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    if not t.cuda.is_available():
        pytest.skip("no CUDA device")
    W.lib()
    yield


# ---------------------------------------------------------------- the generator's two twins agree


@pytest.mark.parametrize("kind,tensor,dtype,count", [
    (synth.KIND_INT4_Q, synth.T_Q, "int8", 1 << 20),
    (synth.KIND_INT4_S, synth.T_S, "int16", 1 << 18),
    (synth.KIND_X, synth.T_X, "int16", 1 << 18),
    (synth.KIND_NVFP4_C, synth.T_C, "uint8", 1 << 20),
    (synth.KIND_NVFP4_S, synth.T_S8, "uint8", 1 << 18)])
def test_device_generator_matches_host(kind, tensor, dtype, count):
    t = torch()
    out = t.empty(count, dtype=getattr(t, dtype), device="cuda")
    synth.device_fill(kind, 17, tensor, out)
    got = out.cpu().numpy()
    idx = np.arange(count, dtype=np.uint64)
    if kind == synth.KIND_INT4_Q:
        want = (synth.codes4(17, tensor, idx).astype(np.int16) - 8).astype(np.int8)
    elif kind == synth.KIND_NVFP4_C:
        want = synth.codes4(17, tensor, idx)
    elif kind == synth.KIND_INT4_S:
        want = synth.to_bf16_bits(0.01 * np.exp(0.25 * synth.normals(17, tensor, idx))).view(np.int16)
    elif kind == synth.KIND_X:
        want = synth.to_bf16_bits(synth.normals(17, tensor, idx)).view(np.int16)
    else:
        want = synth.to_e4m3_bytes(np.abs(synth.normals(17, tensor, idx)) * 0.05)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- dequantisation, bit-exact


def test_dequant_int4_exhaustive_codes_and_scales():
    """All 16 codes x every finite BF16 scale pattern (65,024 rows of K = 128)."""
    t = torch()
    pats = np.array([b for b in range(65536) if (b & 0x7F80) != 0x7F80], dtype=np.uint16)
    N, K = len(pats), 128
    q = np.tile(((np.arange(K) % 16) - 8).astype(np.int8), (N, 1))
    s = pats[:, None]
    codes = t.from_numpy(q).cuda()
    scales = t.from_numpy(s.view(np.int16).copy()).cuda()
    pw, ps = W.pack_on_device("int4", N, K, codes, scales)
    got = bf16_bits(W.dequant("int4", N, K, pw, ps))
    want = oracle.dequant_int4_g128(q, s)
    diff = np.argwhere(got != want)
    assert diff.size == 0, [(int(pats[i]), int(q[i, j]), hex(got[i, j]), hex(want[i, j]))
                            for i, j in diff[:8]]


@pytest.mark.parametrize("g_bits", [0x3B124925, 0x3F800000, 0x3DCCCCCD, 0x4B7FFFFF, 0x0DA24260])
def test_dequant_nvfp4_exhaustive_codes_and_scales(g_bits):
    """All 16 codes x all 254 finite E4M3 scales, for several per-tensor scales."""
    t = torch()
    finite = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], dtype=np.uint8)
    N, K = len(finite), 128
    c = np.tile((np.arange(K) % 16).astype(np.uint8), (N, 1))
    s8 = np.repeat(finite[:, None], K // 16, axis=1)
    g = float(np.array([g_bits], np.uint32).view(np.float32)[0])
    pw, ps = W.pack_on_device("nvfp4", N, K, t.from_numpy(c).cuda(), t.from_numpy(s8).cuda())
    got = bf16_bits(W.dequant("nvfp4", N, K, pw, ps, global_scale=gscale_tensor(g)))
    want = oracle.dequant_nvfp4(c, s8, g)
    diff = np.argwhere(got != want)
    assert diff.size == 0, [(hex(int(finite[i])), int(c[i, j]), hex(got[i, j]), hex(want[i, j]))
                            for i, j in diff[:8]]


@pytest.mark.parametrize("fmt,name", [("int4", "qkv"), ("int4", "down"), ("nvfp4", "o"),
                                      ("nvfp4", "gate_up")])
def test_dequant_full_shapes_sampled_rows(fmt, name):
    K, N = SHAPES[name]
    seed = SEEDS[name] if fmt == "int4" else 6
    t = torch()
    p = synth.device_problem(fmt, seed, 1, N, K)
    pw, ps = W.pack_on_device(fmt, N, K, p["codes"], p["scales"])
    out = W.dequant(fmt, N, K, pw, ps, global_scale=gscale_tensor(p["g"]))
    rows = np.unique(np.concatenate([[0, 15, 16, N - 1], np.random.default_rng(1).integers(0, N, 60)]))
    got = bf16_bits(out[t.from_numpy(rows).cuda()])
    ph = synth.problem(fmt, seed, 1, N, K, rows=rows)
    assert np.array_equal(got, oracle_weights(ph))


@pytest.mark.parametrize("g_bits", [0x3B124925, 0x3F800000, 0x3DCCCCCD, 0x0DA24260])
def test_dequant_fp8_every_code(g_bits):
    """All 254 finite E4M3 weight bytes, for several per-tensor scales."""
    t = torch()
    finite = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], dtype=np.uint8)
    N, K = 16, 256
    c = np.resize(finite, (N, K)).astype(np.uint8)
    g = float(np.array([g_bits], np.uint32).view(np.float32)[0])
    pw, ps = W.pack_on_device("fp8", N, K, t.from_numpy(c).cuda(), None)
    got = bf16_bits(W.dequant("fp8", N, K, pw, ps, global_scale=gscale_tensor(g)))
    want = oracle.dequant_fp8_e4m3(c, g)
    diff = np.argwhere(got != want)
    assert diff.size == 0, [(hex(int(c[i, j])), hex(got[i, j]), hex(want[i, j])) for i, j in diff[:8]]


# ---------------------------------------------------------------- GEMM parity, full oracle


CASES = [  # fmt, M, N, K, seed
    ("int4", 1, 256, 512, 0),          # the tiny configuration
    ("int4", 1, 272, 640, 40),         # 17 bands, ragged against every CTA split
    ("int4", 3, 1000, 1024, 41),       # N not a multiple of 16
    ("int4", 8, 520, 2048, 42),
    ("int4", 9, 304, 1152, 43),
    ("int4", 16, 160, 3072, 44),
    ("int4", 1, 1, 128, 45),           # one output column, one group
    ("int4", 2, 24, 17408, 46),        # long K: several splits
    ("nvfp4", 1, 272, 640, 50),
    ("nvfp4", 5, 1000, 1024, 51),
    ("nvfp4", 9, 304, 1152, 52),
    ("nvfp4", 16, 64, 4096, 53),
    ("nvfp4", 1, 1, 128, 54),
]


@pytest.mark.parametrize("fmt,M,N,K,seed", CASES)
def test_gemm_parity_small(fmt, M, N, K, seed):
    p = synth.problem(fmt, seed, M, N, K)
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm(fmt, codes, scales, x, N, g=p["g"])
    assert_parity(y, p["x"], oracle_weights(p), f"{fmt} M={M} N={N} K={K}")


ROW_COUNTS = [(W.PATH_GEMV, M) for M in (1, 2, 3, 4, 5, 7, 8, 9, 12, 15, 16)] + \
             [(W.PATH_TC, M) for M in (1, 2, 8, 9, 15, 16, 17, 24, 31, 32, 33, 48, 63, 64,
                                       65, 80, 96, 111, 112, 127, 128, 129, 160, 200, 255, 256,
                                       383, 385, 1000, 4096, 8192)]


@pytest.mark.parametrize("path,M", ROW_COUNTS)
def test_gemm_parity_every_row_count(path, M):
    fmt, N, K = "int4", 400, 1536
    p = synth.problem(fmt, 100 + M, M, N, K)
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm(fmt, codes, scales, x, N, path=path)
    assert_parity(y, p["x"], oracle_weights(p), f"path {path} M={M}")


@pytest.mark.parametrize("path,M", [(W.PATH_GEMV, 1), (W.PATH_GEMV, 8), (W.PATH_GEMV, 9),
                                    (W.PATH_GEMV, 16), (W.PATH_TC, 1), (W.PATH_TC, 9),
                                    (W.PATH_TC, 33), (W.PATH_TC, 64), (W.PATH_TC, 80),
                                    (W.PATH_TC, 128), (W.PATH_TC, 129), (W.PATH_TC, 256),
                                    (W.PATH_TC, 1000)])
def test_gemm_parity_every_row_count_nvfp4(path, M):
    fmt, N, K = "nvfp4", 208, 1280
    p = synth.problem(fmt, 200 + M, M, N, K)
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm(fmt, codes, scales, x, N, g=p["g"], path=path)
    assert_parity(y, p["x"], oracle_weights(p), f"nvfp4 M={M}")


FP8_CASES = [  # M, N, K, path (FP8-E4M3 weights, per-tensor scale)
    (1, 272, 640, W.PATH_GEMV), (3, 1000, 1024, W.PATH_GEMV), (8, 520, 2048, W.PATH_GEMV),
    (2, 24, 17408, W.PATH_GEMV), (16, 160, 3072, W.PATH_GEMV), (1, 1, 128, W.PATH_GEMV),
    (9, 304, 1152, W.PATH_TC), (17, 400, 1536, W.PATH_TC), (64, 272, 640, W.PATH_TC),
    (33, 48, 12288, W.PATH_TC), (130, 208, 1280, W.PATH_TC), (1, 16, 128, W.PATH_TC),
]


@pytest.mark.parametrize("M,N,K,path", FP8_CASES)
def test_gemm_parity_fp8(M, N, K, path):
    p = synth.problem("fp8", 400 + M, M, N, K)
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm("fp8", codes, scales, x, N, g=p["g"], path=path)
    assert_parity(y, p["x"], oracle_weights(p), f"fp8 M={M} N={N} K={K} path={path}")


@pytest.mark.parametrize("fmt,M,I,K,path", [("fp8", 1, 48, 640, W.PATH_GEMV),
                                            ("fp8", 12, 96, 4096, W.PATH_GEMV),
                                            ("fp8", 40, 144, 1024, W.PATH_TC),
                                            ("fp8", 9, 48, 17408, W.PATH_TC)])
def test_gate_up_silu_parity_fp8(fmt, M, I, K, path):
    p = synth.problem(fmt, 500 + M, M, 2 * I, K)
    h = _run_gate_up(fmt, p, I, path)
    _assert_gate_up_parity(h, p["x"], oracle_weights(p), f"{fmt} M={M} I={I} K={K}")


@pytest.mark.parametrize("name,M", [("qkv", 1), ("qkv", 16), ("o", 1), ("o", 64), ("qkv", 200)])
def test_gemm_parity_fp8_full_shapes_sampled(name, M):
    K, N = SHAPES[name]
    t = torch()
    seed = SEEDS[name]
    p = synth.device_problem("fp8", seed, M, N, K)
    y, _ = run_gemm("fp8", p["codes"], p["scales"], p["x"], N, g=p["g"])
    rows = np.unique(np.concatenate([[0, 15, 16, N - 1], np.random.default_rng(M).integers(0, N, 40)]))
    ph = synth.problem("fp8", seed, M, N, K, rows=rows)
    assert_parity(y[:, rows], ph["x"], oracle_weights(ph), f"fp8 {name} M={M}")
    del p
    t.cuda.empty_cache()


TC_EDGES = [  # fmt, M, N, K: ragged N against the 256-row tile, the smallest K, chunk edges
    ("int4", 9, 1, 128), ("int4", 64, 17, 128), ("int4", 129, 255, 256), ("int4", 17, 257, 384),
    ("nvfp4", 9, 1, 128), ("nvfp4", 130, 257, 256), ("fp8", 64, 17, 128), ("fp8", 257, 255, 384),
]


@pytest.mark.parametrize("fmt,M,N,K", TC_EDGES)
def test_tensor_core_edges(fmt, M, N, K):
    p = synth.problem(fmt, 600 + M + N, M, N, K)
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm(fmt, codes, scales, x, N, g=p["g"], path=W.PATH_TC)
    assert_parity(y, p["x"], oracle_weights(p), f"TC {fmt} M={M} N={N} K={K}")


# ---------------------------------------------------------------- GEMM parity at the full shapes


FULL = ([("int4", name, 1, SEEDS[name]) for name in SHAPES] +
        [("int4", name, M, 5) for name in ("qkv", "o", "gate_up", "down") for M in (2, 4, 9, 16, 64)] +
        [("nvfp4", name, M, 6) for name in ("qkv", "o", "gate_up", "down") for M in (1, 9, 64)] +
        [("int4", name, M, 7) for name in ("gate_up", "down") for M in (128, 200, 256)] +
        [("nvfp4", name, M, 7) for name in ("o", "gate_up") for M in (96, 256)] +
        [("int4", "gate_up", 1024, 8), ("nvfp4", "down", 640, 8)])


@pytest.mark.parametrize("fmt,name,M,seed", FULL)
def test_gemm_parity_full_shapes_sampled(fmt, name, M, seed):
    K, N = SHAPES[name]
    t = torch()
    p = synth.device_problem(fmt, seed, M, N, K)
    y, _ = run_gemm(fmt, p["codes"], p["scales"], p["x"], N, g=p["g"])
    rows = np.unique(np.concatenate([[0, 7, 8, 15, 16, N - 16, N - 1],
                                     np.random.default_rng(seed + M).integers(0, N, 48)]))
    ph = synth.problem(fmt, seed, M, N, K, rows=rows)
    assert np.array_equal(ph["x"].view(np.int16), p["x"].cpu().numpy())
    assert_parity(y[:, rows], ph["x"], oracle_weights(ph), f"{fmt} {name} M={M}")
    del p
    t.cuda.empty_cache()


# ---------------------------------------------------------------- fused gate/up + SiLU


def _assert_gate_up_parity(h_gpu, x_bits, w_bits, what=""):
    h_ref, gate, up = oracle.gate_up_silu_ref(x_bits, w_bits)
    allowed = oracle.gate_up_silu_allowed(x_bits, w_bits, gate, up)
    err = np.abs(h_gpu - h_ref)
    if not np.all(err <= allowed):
        bad = np.argwhere(err > allowed)[:5]
        detail = [(int(m), int(i), float(h_gpu[m, i]), float(h_ref[m, i]), float(allowed[m, i]))
                  for m, i in bad]
        raise AssertionError(f"{what}: {int((err > allowed).sum())} elements out of tolerance, "
                             f"e.g. {detail}")


def _run_gate_up(fmt, p, I, path=W.PATH_AUTO):
    t = torch()
    codes, scales, x = to_device_problem(p)
    pw, ps = W.pack_on_device(fmt, 2 * I, p["K"], codes, scales)
    h = W.gate_up_silu(fmt, x.view(t.bfloat16), pw, ps, I, global_scale=gscale_tensor(p["g"]),
                       path=path)
    t.cuda.synchronize()
    W.check(W.w4a16_device_status(), "device status")
    return h.float().cpu().numpy().astype(np.float64)


GATE_UP = [  # fmt, M, I, K, path
    ("int4", 1, 48, 640, W.PATH_GEMV), ("int4", 4, 400, 1536, W.PATH_GEMV),
    ("int4", 8, 144, 17408, W.PATH_GEMV),          # long K: split across CTAs
    ("int4", 16, 64, 2048, W.PATH_GEMV), ("nvfp4", 3, 208, 1280, W.PATH_GEMV),
    ("nvfp4", 12, 96, 4096, W.PATH_GEMV), ("nvfp4", 1, 16, 17408, W.PATH_GEMV),
    ("int4", 9, 48, 640, W.PATH_TC), ("int4", 64, 400, 1536, W.PATH_TC),
    ("int4", 17, 144, 17408, W.PATH_TC),           # split K: SiLU in the reduction
    ("int4", 1, 16, 128, W.PATH_TC), ("int4", 200, 272, 1024, W.PATH_TC),
    ("nvfp4", 33, 208, 1280, W.PATH_TC), ("nvfp4", 128, 160, 2048, W.PATH_TC),
    ("nvfp4", 40, 48, 12288, W.PATH_TC), ("int4", 1000, 144, 384, W.PATH_TC),
    ("int4", 5, 32, 512, W.PATH_AUTO), ("nvfp4", 70, 64, 512, W.PATH_AUTO),
]


@pytest.mark.parametrize("fmt,M,I,K,path", GATE_UP)
def test_gate_up_silu_parity(fmt, M, I, K, path):
    p = synth.problem(fmt, 300 + M + I, M, 2 * I, K)
    h = _run_gate_up(fmt, p, I, path)
    _assert_gate_up_parity(h, p["x"], oracle_weights(p), f"{fmt} M={M} I={I} K={K} path={path}")


@pytest.mark.parametrize("fmt,M", [("int4", 1), ("int4", 9), ("int4", 64), ("nvfp4", 1),
                                   ("nvfp4", 64), ("int4", 256)])
def test_gate_up_silu_full_shape_sampled(fmt, M):
    K, N = SHAPES["gate_up"]
    I = N // 2
    t = torch()
    seed = SEEDS["gate_up"]
    p = synth.device_problem(fmt, seed, M, N, K)
    pw, ps = W.pack_on_device(fmt, N, K, p["codes"], p["scales"])
    h = W.gate_up_silu(fmt, p["x"].view(t.bfloat16), pw, ps, I, global_scale=gscale_tensor(p["g"]))
    t.cuda.synchronize()
    cols = np.unique(np.concatenate([[0, 15, 16, 127, 128, I - 1],
                                     np.random.default_rng(M).integers(0, I, 40)]))
    ph = synth.problem(fmt, seed, M, N, K, rows=np.concatenate([cols, I + cols]))
    hs = h[:, t.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    _assert_gate_up_parity(hs, ph["x"], oracle_weights(ph), f"{fmt} gate_up M={M}")
    del p, pw, ps, h
    t.cuda.empty_cache()


def test_gate_up_silu_matches_the_unfused_pair():
    # the fused layer against SiLU / product applied on the host to the two
    # halves of the plain matmul: both within tolerance of each other
    t = torch()
    fmt, M, I, K = "int4", 6, 272, 1024
    p = synth.problem(fmt, 77, M, 2 * I, K)
    codes, scales, x = to_device_problem(p)
    pw, ps = W.pack_on_device(fmt, 2 * I, K, codes, scales)
    xb = x.view(t.bfloat16)
    y = W.gemm(fmt, xb, pw, ps, 2 * I).float().cpu().numpy().astype(np.float64)
    h = W.gate_up_silu(fmt, xb, pw, ps, I).float().cpu().numpy().astype(np.float64)
    w = oracle_weights(p)
    _, gate, up = oracle.gate_up_silu_ref(p["x"], w)
    allowed = oracle.gate_up_silu_allowed(p["x"], w, gate, up)
    assert np.all(np.abs(h - oracle.silu(y[:, :I]) * y[:, I:]) <= 2 * allowed)


# ---------------------------------------------------------------- invariants and edge cases


def _packed(fmt, p):
    codes, scales, x = to_device_problem(p)
    pw, ps = W.pack_on_device(fmt, p["N"], p["K"], codes, scales)
    return pw, ps, x


def test_one_hot_selects_dequantised_column_bit_exact():
    t = torch()
    for fmt in ("int4", "nvfp4"):
        N, K = 96, 640
        p = synth.problem(fmt, 61, 1, N, K)
        pw, ps, _ = _packed(fmt, p)
        g = gscale_tensor(p["g"])
        wd = bf16_bits(W.dequant(fmt, N, K, pw, ps, global_scale=g))
        for k in (0, 5, 127, 128, 333, K - 1):
            x = t.zeros((1, K), dtype=t.bfloat16, device="cuda")
            x[0, k] = 1.0
            y = W.gemm(fmt, x, pw, ps, N, global_scale=g)
            t.cuda.synchronize()
            # y = 1 * W_deq[n][k] + (+0) * the rest: the same value, and the same
            # bits except that a -0 weight sums to +0
            assert np.array_equal(formats.bf16_to_f64(bf16_bits(y)[0]),
                                  formats.bf16_to_f64(wd[:, k])), (fmt, k)
            nz = (wd[:, k] & 0x7FFF) != 0
            assert np.array_equal(bf16_bits(y)[0][nz], wd[nz, k]), (fmt, k)


def test_doubling_x_doubles_y_bit_exact_and_zero_scales_give_zero():
    t = torch()
    for fmt in ("int4", "nvfp4"):
        for M in (1, 9, 64):
            N, K = 128, 1024
            p = synth.problem(fmt, 62 + M, M, N, K)
            pw, ps, x = _packed(fmt, p)
            g = gscale_tensor(p["g"])
            xb = x.view(t.bfloat16)
            y1 = bf16_bits(W.gemm(fmt, xb, pw, ps, N, global_scale=g))
            y2 = bf16_bits(W.gemm(fmt, xb * 2, pw, ps, N, global_scale=g))
            v1 = formats.bf16_to_f64(y1)
            assert np.array_equal(formats.bf16_to_f64(y2), 2 * v1), (fmt, M)
            zs = t.zeros_like(t.from_numpy(np.ascontiguousarray(
                p["scales"].view(np.int16) if p["scales"].dtype == np.uint16 else p["scales"])).cuda())
            codes, _, _ = to_device_problem(p)
            pw0, ps0 = W.pack_on_device(fmt, N, K, codes, zs)
            y0 = W.gemm(fmt, xb, pw0, ps0, N, global_scale=g).float().cpu().numpy()
            assert np.all(y0 == 0), (fmt, M)


def test_output_guard_bands_and_full_coverage():
    t = torch()
    for fmt, M, N, K in (("int4", 3, 50, 640), ("int4", 8, 24, 17408), ("nvfp4", 9, 40, 512),
                         ("int4", 64, 33, 384), ("int4", 200, 33, 384), ("nvfp4", 129, 40, 512)):
        p = synth.problem(fmt, 70 + M, M, N, K)
        pw, ps, x = _packed(fmt, p)
        pad = 64
        buf = t.full((M * N + 2 * pad,), float("nan"), dtype=t.bfloat16, device="cuda")
        sentinel = t.tensor(12345.0, dtype=t.bfloat16)
        buf[:pad] = sentinel
        buf[-pad:] = sentinel
        y = buf[pad:pad + M * N].view(M, N)
        W.gemm(fmt, x.view(t.bfloat16), pw, ps, N, global_scale=gscale_tensor(p["g"]), y=y)
        t.cuda.synchronize()
        host = buf.float().cpu().numpy()
        assert np.all(host[:pad] == 12352.0) and np.all(host[-pad:] == 12352.0), (fmt, M, N, K)
        assert not np.any(np.isnan(host[pad:-pad])), (fmt, M, N, K)


def test_repeated_calls_are_bit_identical():
    # fixed reduction orders everywhere (split-K partials are added in split
    # order on both paths), so repeated calls agree bit for bit
    t = torch()
    for fmt, M, N, K in (("int4", 8, 5120, 17408), ("int4", 1, 17408, 5120), ("nvfp4", 9, 1024, 6144),
                         ("int4", 64, 5120, 6144), ("int4", 200, 2048, 5120), ("fp8", 33, 1024, 17408)):
        p = synth.device_problem(fmt, 80, M, N, K)
        pw, ps = W.pack_on_device(fmt, N, K, p["codes"], p["scales"])
        g = gscale_tensor(p["g"])
        xb = p["x"].view(t.bfloat16)
        ys = [bf16_bits(W.gemm(fmt, xb, pw, ps, N, global_scale=g)) for _ in range(3)]
        assert all(np.array_equal(ys[0], yy) for yy in ys[1:]), (fmt, M, N, K)
        hs = [bf16_bits(W.gate_up_silu(fmt, xb, pw, ps, N // 2, global_scale=g)) for _ in range(2)]
        assert np.array_equal(hs[0], hs[1]), (fmt, M, N, K, "fused")


def test_golden_examples_on_gpu():
    t = torch()
    d = json.load(open(os.path.join(GOLDEN, "int4_worked_example.json")))
    k = np.arange(128)
    q = np.stack([(k % 16) - 8, 7 - (k % 16)]).astype(np.int8)
    s = np.array(d["inputs"]["scale_bits"], dtype=np.uint16)
    pw, ps = W.pack_on_device("int4", 2, 128, t.from_numpy(q).cuda(),
                              t.from_numpy(s.view(np.int16).copy()).cuda())
    wd = bf16_bits(W.dequant("int4", 2, 128, pw, ps))
    assert [int(v) for v in wd[0, :16]] == [int(h, 16) for h in d["expected"]["w_row0_hex_k0_to_15"]]
    x = t.zeros((1, 128), dtype=t.bfloat16, device="cuda")
    x[0, :16] = 1.0
    y = W.gemm("int4", x, pw, ps, 2).float().cpu().numpy()[0]
    assert list(y) == d["expected"]["y"]
    d = json.load(open(os.path.join(GOLDEN, "nvfp4_worked_example.json")))
    c = np.tile(np.arange(16, dtype=np.uint8), (2, 8))
    s8 = np.repeat(np.array(d["inputs"]["scale_e4m3"], dtype=np.uint8), 8, axis=1)
    pw, ps = W.pack_on_device("nvfp4", 2, 128, t.from_numpy(c).cuda(), t.from_numpy(s8).cuda())
    g = gscale_tensor(1.0)
    wd = bf16_bits(W.dequant("nvfp4", 2, 128, pw, ps, global_scale=g))
    assert [int(v) for v in wd[0, :16]] == [int(h, 16) for h in d["expected"]["w_row0_hex_k0_to_15"]]
    x = t.zeros((1, 128), dtype=t.bfloat16, device="cuda")
    x[0, :8] = 1.0
    y = W.gemm("nvfp4", x, pw, ps, 2, global_scale=g).float().cpu().numpy()[0]
    assert list(y) == d["expected"]["y"]


def test_bounded_wait_runs_out_reports_a_timeout_and_leaves_the_context_usable():
    # a wait on an mbarrier that nothing arrives at gives up after its bound
    # (about two seconds), records W4A16_ERR_TIMEOUT and the kernel exits
    assert W.w4a16_selftest_wait_timeout() == W.OK
    assert W.w4a16_device_status() == W.OK          # the word was read and cleared
    p = synth.problem("int4", 11, 3, 64, 256)      # the context still computes correctly
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm("int4", codes, scales, x, 64)
    assert_parity(y, p["x"], oracle_weights(p), "after the timeout self-test")


def test_device_status_is_clean():
    assert W.w4a16_device_status() == W.OK


# ---------------------------------------------------------------- chained launches
# Every GEMV and tensor-core launch (and the FP16 rescale of the NVFP4 and
# FP8 tensor-core paths) lets the next kernel on the stream start early
# (programmatic dependent launch) and waits for the previous one only before
# it reads the activations.  A chain whose layers feed each other, issued
# back to back with no host synchronisation (eagerly and as a CUDA graph),
# checks that each layer reads its input only after the previous layer wrote
# it: every layer is compared with the oracle applied to the previous layer's
# GPU output.


def _chain_layers(fmt, dims, seed):
    layers = []
    for i, (K, N) in enumerate(zip(dims[:-1], dims[1:])):
        p = synth.problem(fmt, seed + i, 1, N, K)
        codes, scales, _ = to_device_problem(p)
        pw, ps = W.pack_on_device(fmt, N, K, codes, scales)
        layers.append((K, N, pw, ps, gscale_tensor(p["g"]), oracle_weights(p)))
    return layers


@pytest.mark.parametrize("fmt,M,path", [("int4", 1, W.PATH_GEMV), ("int4", 4, W.PATH_GEMV),
                                        ("int4", 9, W.PATH_AUTO), ("nvfp4", 2, W.PATH_GEMV),
                                        ("nvfp4", 9, W.PATH_TC), ("fp8", 16, W.PATH_TC)])
@pytest.mark.parametrize("graph", [False, True])
def test_chained_layers_read_their_inputs_after_they_are_written(fmt, M, path, graph):
    t = torch()
    dims = [1024, 2048, 1536, 3072, 1024, 2048, 1024]
    layers = _chain_layers(fmt, dims, 300 + M)
    x0 = synth.problem(fmt, 399, M, 256, dims[0])["x"]
    bufs = [t.from_numpy(np.ascontiguousarray(x0.view(np.int16))).cuda().view(t.bfloat16)]
    for K, N, *_ in layers:
        bufs.append(t.full((M, N), float("nan"), dtype=t.bfloat16, device="cuda"))
    s = t.cuda.Stream()

    def run():
        for i, (K, N, pw, ps, g, _) in enumerate(layers):
            W.gemm(fmt, bufs[i], pw, ps, N, global_scale=g, y=bufs[i + 1], path=path, stream=s)

    with t.cuda.stream(s):
        if graph:
            run()                       # plans and workspace outside the capture
            s.synchronize()
            for b in bufs[1:]:
                b.fill_(float("nan"))
            gr = t.cuda.CUDAGraph()
            with t.cuda.graph(gr, stream=s):
                run()
            gr.replay()
        else:
            run()
    s.synchronize()
    W.check(W.w4a16_device_status(s), "device status")
    for i, (K, N, pw, ps, g, wref) in enumerate(layers):
        x_in = bf16_bits(bufs[i])
        y = bufs[i + 1].float().cpu().numpy().astype(np.float64)
        assert not np.isnan(y).any(), (fmt, M, i)
        assert_parity(y, x_in, wref, f"{fmt} M={M} layer {i}")


# ---------------------------------------------------------------- edge values through the GEMMs
# Scales that are negative, subnormal, zero, very large or very small; groups
# whose codes are all zero; activation rows spanning up to 2^-24 .. 2^24 (see
# synth.adversarial_problem).  Both paths, every format, element by element
# against the oracle at the accuracy contract.

EDGE_CASES = (
    [("int4", reg, W.PATH_GEMV, M, 264, 1024) for reg in ("extreme", "wide") for M in (1, 3, 8, 16)] +
    [("int4", reg, W.PATH_TC, M, 264, 1024) for reg in ("extreme", "wide") for M in (9, 64, 130)] +
    [("int4", reg, path, M, 40, 17408) for reg in ("extreme", "wide")
     for path, M in ((W.PATH_GEMV, 2), (W.PATH_TC, 17))] +
    [("nvfp4", reg, W.PATH_GEMV, M, 208, 1280) for reg in ("extreme", "wide") for M in (1, 5, 16)] +
    [("nvfp4", reg, W.PATH_TC, M, 208, 1280) for reg in ("extreme", "wide") for M in (9, 64)] +
    [("nvfp4", reg, path, M, 48, 12288) for reg in ("extreme", "wide")
     for path, M in ((W.PATH_GEMV, 3), (W.PATH_TC, 40))] +
    [("fp8", reg, W.PATH_GEMV, M, 200, 1536) for reg in ("extreme", "wide") for M in (2, 12)] +
    [("fp8", reg, W.PATH_TC, M, 200, 1536) for reg in ("extreme", "wide") for M in (33, 64)])


@pytest.mark.parametrize("fmt,regime,path,M,N,K", EDGE_CASES)
def test_gemm_parity_edge_values(fmt, regime, path, M, N, K):
    p = synth.adversarial_problem(fmt, 700 + M + K % 97, M, N, K, regime)
    codes, scales, x = to_device_problem(p)
    y, _ = run_gemm(fmt, codes, scales, x, N, g=p["g"], path=path)
    w = oracle_weights(p)
    assert np.isfinite(oracle.gemm_ref(p["x"], w)).all()
    assert_parity(y, p["x"], w, f"edge {fmt} {regime} path={path} M={M} N={N} K={K}")


# The fused layer multiplies two matmul outputs, so the "extreme" int4 scales
# (up to 2^100) would square past the BF16 range: the int4 cases use the
# "wide" inputs, and every case checks that h itself is representable.
@pytest.mark.parametrize("fmt,regime,path,M,I,K", [
    ("int4", "wide", W.PATH_GEMV, 4, 64, 2048), ("int4", "wide", W.PATH_TC, 24, 144, 1024),
    ("nvfp4", "extreme", W.PATH_TC, 64, 48, 1280), ("nvfp4", "extreme", W.PATH_GEMV, 3, 48, 1280),
    ("fp8", "wide", W.PATH_GEMV, 7, 96, 1536)])
def test_gate_up_silu_parity_edge_values(fmt, regime, path, M, I, K):
    p = synth.adversarial_problem(fmt, 750 + M, M, 2 * I, K, regime)
    h_ref, _, _ = oracle.gate_up_silu_ref(p["x"], oracle_weights(p))
    assert np.abs(h_ref).max() < 3.38e38                 # below the largest BF16 value
    h = _run_gate_up(fmt, p, I, path)
    _assert_gate_up_parity(h, p["x"], oracle_weights(p), f"edge gate/up {fmt} {regime} M={M}")


# ---------------------------------------------------------------- the output projection
# The whole-stack sweep's 5120 -> 248,320 int4 output projection (layer seed
# 71): the largest packed weight (636 MB) and output the library addresses.


@pytest.mark.parametrize("M,path", [(1, W.PATH_AUTO), (16, W.PATH_AUTO), (16, W.PATH_TC),
                                    (64, W.PATH_AUTO)])
def test_gemm_parity_output_projection_sampled(M, path):
    K, N, seed = 5120, 248320, 71
    t = torch()
    p = synth.device_problem("int4", seed, M, N, K)
    y, (pw, ps, _) = run_gemm("int4", p["codes"], p["scales"], p["x"], N, path=path)
    del p
    rows = np.unique(np.concatenate([[0, 15, 16, 255, 256, N - 257, N - 16, N - 1],
                                     np.random.default_rng(M + path).integers(0, N, 48)]))
    ph = synth.problem("int4", seed, M, N, K, rows=rows)
    assert_parity(y[:, rows], ph["x"], oracle_weights(ph), f"output projection M={M} path={path}")
    del pw, ps
    t.cuda.empty_cache()
