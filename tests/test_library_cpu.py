"""The C-ABI library without a GPU: symbols, host packer, argument checks."""

from __future__ import annotations

import os
import re

import numpy as np
import pytest

import synth
from bit_weight_only_dequant_b200 import w4a16 as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "w4a16.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a16_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = W.lib()
    names = _declared_functions()
    assert "w4a16_gemm" in names and "w4a16_dequant" in names
    for name in names:
        assert hasattr(lib, name), name
    assert W.w4a16_version() >= 100


def test_status_strings():
    for st in (W.OK, W.ERR_ARG, W.ERR_SHAPE, W.ERR_ALIGN, W.ERR_DEVICE, W.ERR_CUDA,
               W.ERR_TIMEOUT, W.ERR_NOMEM):
        assert W.status_string(st).startswith("W4A16_")


def test_packed_sizes():
    assert W.w4a16_packed_weight_bytes(0, 8192, 5120) == 8192 * 5120 // 2
    assert W.w4a16_packed_scale_bytes(0, 8192, 5120) == 8192 * 40 * 2
    assert W.w4a16_packed_scale_bytes(1, 8192, 5120) == 8192 * 320
    assert W.w4a16_packed_weight_bytes(0, 17, 128) == 32 * 64          # rows padded to 16
    assert W.w4a16_packed_weight_bytes(0, 16, 100) == 0                 # K not a multiple of 128
    assert W.w4a16_packed_weight_bytes(4, 16, 128) == 0                 # bad format
    assert W.w4a16_packed_weight_bytes(2, 8192, 5120) == 8192 * 5120    # FP8: a byte per weight
    assert W.w4a16_packed_scale_bytes(2, 8192, 5120) == 0               # per-tensor scale only
    assert W.w4a16_packed_weight_bytes(2, 17, 128) == 32 * 128
    # block-scaled W4A4 layout: no row padding for the codes, scale atoms of 128 rows x 64 k
    assert W.w4a16_packed_weight_bytes(3, 17, 128) == 17 * 64
    assert W.w4a16_packed_scale_bytes(3, 17, 128) == 1 * 2 * 512
    assert W.w4a16_packed_scale_bytes(3, 8192, 5120) == 64 * 80 * 512 == 8192 * 320
    assert W.w4a16_packed_scale_bytes(3, 129, 256) == 2 * 4 * 512


@pytest.mark.parametrize("fmt,N,K", [("int4", 16, 128), ("int4", 37, 384), ("nvfp4", 16, 128),
                                     ("nvfp4", 45, 256), ("fp8", 16, 128), ("fp8", 45, 384),
                                     ("nvfp4_bs", 45, 256), ("nvfp4_bs", 130, 384)])
def test_host_pack_round_trip(fmt, N, K):
    p = synth.problem("nvfp4" if fmt == "nvfp4_bs" else fmt, 7, 1, N, K)
    f = W.FMTS[fmt]
    w = np.zeros(W.w4a16_packed_weight_bytes(f, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(f, N, K), np.uint8)
    assert W.w4a16_pack_host(f, N, K, p["codes"], p["scales"], w, s) == W.OK
    codes = np.zeros_like(p["codes"])
    scales = None if p["scales"] is None else np.zeros_like(p["scales"])
    assert W.w4a16_unpack_host(f, N, K, w, s, codes, scales) == W.OK
    assert np.array_equal(codes, p["codes"])
    if scales is not None:
        assert np.array_equal(scales, p["scales"])


def test_host_pack_fp8_layout_and_nan_rejection():
    # FP8: 16 x 32 tiles of 512 bytes; lane 4g + t, k16 sub-block j, words
    # 2j (P0, P1) and 2j + 1 (P2, P3), a byte per element (restated here)
    N, K = 32, 128
    codes = (np.arange(N * K) % 0x7E + 1).astype(np.uint8).reshape(N, K)   # no NaN byte
    w = np.zeros(W.w4a16_packed_weight_bytes(2, N, K), np.uint8)
    assert W.w4a16_pack_host(2, N, K, codes, None, w, None) == W.OK
    for n in range(N):
        for k in range(K):
            nt, kt, r, kk = n // 16, k // 32, n % 16, k % 32
            g, hi, j, kin = r % 8, r // 8, kk // 16, kk % 16
            t, e = kin // 4, kin % 4
            pair, second = hi + 2 * (e // 2), e % 2
            off = ((nt * (K // 32) + kt) * 512 + (4 * g + t) * 16 + (2 * j + pair // 2) * 4
                   + 2 * (pair % 2) + second)
            assert w[off] == codes[n, k], (n, k)
    bad = codes.copy()
    bad[3, 77] = 0xFF
    assert W.w4a16_pack_host(2, N, K, bad, None, w, None) == W.ERR_ARG


def _layout_position(fmt, n, k, K):
    """The packed position of (n, k) restated from the layout description."""
    nt, kb = n // 16, k // 64
    r, kk = n % 16, k % 64
    g, hi = r % 8, r // 8
    j, kin = kk // 16, kk % 16
    t, e = kin // 4, kin % 4
    pair = hi + 2 * (e // 2)
    second = e % 2
    nib = pair + 4 * second if fmt == 0 else 2 * pair + second
    word = (nt * (K // 64) + kb) * 512 + (4 * g + t) * 16 + 4 * j
    return word + nib // 2, 4 * (nib % 2)


@pytest.mark.parametrize("fmt", [0, 1])
def test_host_pack_matches_the_documented_layout(fmt):
    N, K = 32, 256
    codes = np.zeros((N, K), dtype=np.int8 if fmt == 0 else np.uint8)
    rng = np.random.default_rng(3)
    picks = [(int(rng.integers(N)), int(rng.integers(K))) for _ in range(40)]
    for n, k in picks:
        codes[n, k] = 5 if fmt == 0 else 11
    scales = np.zeros((N, K // (128 if fmt == 0 else 16)), dtype=np.uint16 if fmt == 0 else np.uint8)
    w = np.zeros(W.w4a16_packed_weight_bytes(fmt, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(fmt, N, K), np.uint8)
    assert W.w4a16_pack_host(fmt, N, K, codes, scales, w, s) == W.OK
    zero = 8 if fmt == 0 else 0                  # the stored nibble of value 0
    expect = np.zeros_like(w)
    for n in range(N):
        for k in range(K):
            b, sh = _layout_position(fmt, n, k, K)
            v = (int(codes[n, k]) + 8) & 15 if fmt == 0 else int(codes[n, k])
            expect[b] |= v << sh
    assert np.array_equal(w, expect)
    assert zero in (0, 8)


def test_host_pack_scale_layout():
    N, K = 32, 256
    q = np.zeros((N, K), np.int8)
    sc = (np.arange(N * 2, dtype=np.uint16) + 0x3F00).reshape(N, 2)
    w = np.zeros(W.w4a16_packed_weight_bytes(0, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(0, N, K), np.uint8)
    assert W.w4a16_pack_host(0, N, K, q, sc, w, s) == W.OK
    s16 = s.view(np.uint16)
    for n in range(N):
        for gi in range(2):
            off = ((n // 16) * 2 + gi) * 32 + (n % 8) * 4 + (n % 16 // 8) * 2
            assert s16[off // 2] == sc[n, gi]
    c = np.zeros((N, K), np.uint8)
    s8 = (np.arange(N * 16) % 0x70).astype(np.uint8).reshape(N, 16)
    w = np.zeros(W.w4a16_packed_weight_bytes(1, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(1, N, K), np.uint8)
    assert W.w4a16_pack_host(1, N, K, c, s8, w, s) == W.OK
    for n in range(N):
        for gi in range(16):
            off = ((n // 16) * 4 + gi // 4) * 64 + (n % 8) * 8 + (gi % 4) * 2 + (n % 16) // 8
            assert s[off] == s8[n, gi]


def test_host_pack_rejects_out_of_range():
    N, K = 16, 128
    w = np.zeros(W.w4a16_packed_weight_bytes(0, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(0, N, K), np.uint8)
    q = np.zeros((N, K), np.int8)
    q[3, 5] = 8
    assert W.w4a16_pack_host(0, N, K, q, np.zeros((N, 1), np.uint16), w, s) == W.ERR_ARG
    nanscale = np.full((N, 1), 0x7FC0, np.uint16)
    assert W.w4a16_pack_host(0, N, K, np.zeros((N, K), np.int8), nanscale, w, s) == W.ERR_ARG
    w = np.zeros(W.w4a16_packed_weight_bytes(1, N, K), np.uint8)
    s = np.zeros(W.w4a16_packed_scale_bytes(1, N, K), np.uint8)
    c = np.zeros((N, K), np.uint8)
    c[0, 0] = 16
    assert W.w4a16_pack_host(1, N, K, c, np.zeros((N, 8), np.uint8), w, s) == W.ERR_ARG
    assert W.w4a16_pack_host(1, N, K, np.zeros((N, K), np.uint8), np.full((N, 8), 0x7F, np.uint8),
                             w, s) == W.ERR_ARG


def test_argument_validation_before_any_device_call():
    x = w = s = y = 1 << 20          # fake, aligned, never dereferenced
    assert W.w4a16_gemm(0, 0, 16, 128, x, w, s, None, y, 0) == W.ERR_SHAPE       # M = 0
    assert W.w4a16_gemm(0, 8193, 16, 128, x, w, s, None, y, 0) == W.ERR_SHAPE    # M > 8192
    assert W.w4a16_gemm_ex(W.PATH_GEMV, 0, 17, 16, 128, x, w, s, None, y, 0) == W.ERR_SHAPE
    assert W.w4a16_gemm(0, 1, 16, 100, x, w, s, None, y, 0) == W.ERR_SHAPE       # K % 128
    assert W.w4a16_gemm(0, 1, 0, 128, x, w, s, None, y, 0) == W.ERR_SHAPE        # N = 0
    assert W.w4a16_gemm(3, 1, 16, 128, x, w, s, None, y, 0) == W.ERR_ARG         # format
    assert W.w4a16_gemm(0, 1, 16, 128, None, w, s, None, y, 0) == W.ERR_ARG      # null x
    assert W.w4a16_gemm(0, 1, 16, 128, x, w, s, 1 << 21, y, 0) == W.ERR_ARG      # g for int4
    assert W.w4a16_gemm(1, 1, 16, 128, x, w, s, None, y, 0) == W.ERR_ARG         # no g for nvfp4
    assert W.w4a16_gemm(2, 1, 16, 128, x, w, None, None, y, 0) == W.ERR_ARG      # no g for fp8
    assert W.w4a16_gemm(0, 1, 16, 128, x, w, None, None, y, 0) == W.ERR_ARG      # no scales, int4
    assert W.w4a16_gemm(0, 1, 16, 128, x + 2, w, s, None, y, 0) == W.ERR_ALIGN
    assert W.w4a16_gemm_ex(7, 0, 1, 16, 128, x, w, s, None, y, 0) == W.ERR_ARG   # bad path
    assert W.w4a16_dequant(0, 16, 128, w, s, None, y + 8, 0) == W.ERR_ALIGN
    assert W.w4a16_pack(0, 16, 100, x, s, w, s, 0) == W.ERR_SHAPE


def test_gate_up_silu_argument_validation():
    x = w = s = h = 1 << 20          # fake, aligned, never dereferenced
    assert W.w4a16_gemm_gate_up_silu(0, 1, 24, 128, x, w, s, None, h, 0) == W.ERR_SHAPE   # I % 16
    assert W.w4a16_gemm_gate_up_silu(0, 1, 0, 128, x, w, s, None, h, 0) == W.ERR_SHAPE    # I = 0
    assert W.w4a16_gemm_gate_up_silu(0, 0, 16, 128, x, w, s, None, h, 0) == W.ERR_SHAPE   # M = 0
    assert W.w4a16_gemm_gate_up_silu(0, 8193, 16, 128, x, w, s, None, h, 0) == W.ERR_SHAPE
    assert W.w4a16_gemm_gate_up_silu(0, 1, 16, 100, x, w, s, None, h, 0) == W.ERR_SHAPE   # K % 128
    assert W.w4a16_gemm_gate_up_silu(5, 1, 16, 128, x, w, s, None, h, 0) == W.ERR_ARG     # format
    assert W.w4a16_gemm_gate_up_silu(1, 1, 16, 128, x, w, s, None, h, 0) == W.ERR_ARG     # no g
    assert W.w4a16_gemm_gate_up_silu(0, 1, 16, 128, x, w, s, None, h + 4, 0) == W.ERR_ALIGN
    assert W.w4a16_gemm_gate_up_silu_ex(9, 0, 1, 16, 128, x, w, s, None, h, 0) == W.ERR_ARG
    assert W.w4a16_gemm_gate_up_silu_ex(W.PATH_GEMV, 0, 17, 16, 128, x, w, s, None, h, 0) == W.ERR_SHAPE


def test_dispatcher_path_table():
    for M in range(1, W.MAX_M + 1):
        path = W.w4a16_gemm_path(0, M, 5120, 5120)
        assert path in (W.PATH_GEMV, W.PATH_TC)
        assert M <= 16 or path == W.PATH_TC
    assert W.w4a16_gemm_path(0, 1, 17408, 5120) == W.PATH_GEMV
    assert W.w4a16_gemm_path(0, 8, 5120, 6144) == W.PATH_GEMV
    assert W.w4a16_gemm_path(0, 9, 5120, 6144) == W.PATH_TC      # narrow int4 layer
    assert W.w4a16_gemm_path(0, 16, 8192, 5120) == W.PATH_TC
    assert W.w4a16_gemm_path(0, 16, 34816, 5120) == W.PATH_GEMV  # wide int4 layer
    assert W.w4a16_gemm_path(1, 16, 5120, 17408) == W.PATH_TC    # NVFP4, narrow layer
    assert W.w4a16_gemm_path(1, 16, 34816, 5120) == W.PATH_GEMV  # NVFP4, wide layer
    assert W.w4a16_gemm_path(0, 17, 34816, 5120) == W.PATH_TC
    assert W.w4a16_gemm_path(0, 64, 34816, 5120) == W.PATH_TC
    assert W.w4a16_gemm_path(0, 65, 5120, 5120) == W.PATH_TC
    assert W.w4a16_gemm_path(1, 256, 17408, 5120) == W.PATH_TC
    assert W.w4a16_gemm_path(0, 8192, 5120, 5120) == W.PATH_TC
    assert W.w4a16_gemm_path(0, 8193, 5120, 5120) == W.ERR_SHAPE


DECODE = [(5120, 8192), (6144, 5120), (5120, 34816), (17408, 5120), (5120, 17408), (128, 16),
          (384, 1000), (17408, 24), (12288, 48)]


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("fuse", [0, 1])
def test_gemv_plans_are_consistent(fmt, fuse):
    # every GEMV plan the planner hands out covers K exactly with whole
    # 128-groups, uses an instantiated ring depth and fits in shared memory
    for K, N in DECODE:
        if fuse and N % 32:
            continue
        for M in (1, 2, 5, 8, 9, 12, 16):
            r, (S, kslice, ctas, mt, wn, wk, depth, ngp, smem) = W.w4a16_plan(W.PATH_GEMV, fmt, M, N, K,
                                                                              fuse)
            assert r == W.PATH_GEMV, (fmt, fuse, M, N, K, r)
            assert S >= 1 and kslice % 128 == 0 and S * kslice >= K > (S - 1) * kslice
            assert mt == (1 if M <= 8 else 2)
            assert wn * wk == 16 and wn & (wn - 1) == 0
            assert depth in ((2, 3, 4) if (fuse or fmt == 2) else (2, 3, 4, 5, 6, 8))
            assert ngp % depth == 0 and ngp * wk * 128 >= min(kslice, K)
            bands = (N // 2 if fuse else N + 15) // 16
            assert 1 <= ctas <= bands and ctas * S <= 148
            assert 0 < smem <= 227 * 1024


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("fuse", [0, 1])
def test_tensor_core_plans_are_consistent(fmt, fuse):
    for K, N in DECODE:
        if fuse and N % 32:
            continue
        for M in (1, 9, 16, 17, 64, 65, 128, 129, 200, 256, 1000, 8192):
            r, (chunks, rows, mpad, S, kbs, units, grid, smem, _) = W.w4a16_plan(W.PATH_TC, fmt, M, N,
                                                                                 K, fuse)
            assert r == W.PATH_TC
            assert chunks * rows >= M > (chunks - 1) * rows and rows <= 128
            assert mpad % 16 == 0 and rows <= mpad <= 128 and mpad - rows < 16
            assert S >= 1 and kbs % 2 == 0 and S * kbs * 64 >= K > (S - 1) * kbs * 64
            tiles = (N // 2 + 127) // 128 if fuse else (N + 255) // 256
            assert units == tiles * chunks * S
            assert 1 <= grid <= min(units, 148)
            assert 120 * 1024 <= smem <= 227 * 1024


def test_plans_follow_the_dispatcher():
    assert W.w4a16_plan(W.PATH_AUTO, 0, 1, 17408, 5120)[0] == W.PATH_GEMV
    assert W.w4a16_plan(W.PATH_AUTO, 0, 64, 34816, 5120)[0] == W.PATH_TC
    assert W.w4a16_plan(W.PATH_GEMV, 0, 17, 16, 128)[0] == W.ERR_SHAPE
    assert W.w4a16_plan(W.PATH_TC, 0, 1, 24, 128, fuse=1)[0] == W.ERR_SHAPE      # 2I not a multiple of 32


def test_host_pack_block_scaled_layout():
    # W4A16_FMT_NVFP4_BS, restated from its description: codes [N][K/2] with
    # k = 2j in the low nibble of byte j; scales in 512-byte atoms per (128-row
    # tile, 64-k block), row r = a + 32 b and 16-block j at byte 16 a + 4 b + j
    N, K = 150, 256
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    s8 = rng.integers(0, 0x7F, size=(N, K // 16)).astype(np.uint8)
    w = np.zeros(W.w4a16_packed_weight_bytes(3, N, K), np.uint8)
    s = np.full(W.w4a16_packed_scale_bytes(3, N, K), 0xAA, np.uint8)
    assert W.w4a16_pack_host(3, N, K, codes, s8, w, s) == W.OK
    assert np.array_equal(w, (codes[:, 0::2] | (codes[:, 1::2] << 4)).reshape(-1))
    expect = np.zeros_like(s)
    for n in range(N):
        t, r = divmod(n, 128)
        for gi in range(K // 16):
            expect[(t * (K // 64) + gi // 4) * 512 + 16 * (r % 32) + 4 * (r // 32) + gi % 4] = s8[n, gi]
    assert np.array_equal(s, expect)          # rows past N of the last tile hold 0
    bad = s8.copy()
    bad[5, 3] = 0x7F
    assert W.w4a16_pack_host(3, N, K, codes, bad, w, s) == W.ERR_ARG


def test_block_scaled_plan_invariants():
    out = np.zeros(9, np.int32)
    for M, N, K in [(1, 8192, 5120), (9, 5120, 6144), (64, 34816, 5120), (64, 5120, 17408),
                    (1, 1, 256), (200, 300, 1024), (8192, 1000, 512), (129, 256, 128)]:
        r = W.lib().w4a16_plan(W.PATH_BS, 3, M, N, K, 0, 148, out.ctypes.data, 9)
        assert r == W.PATH_BS, (M, N, K, r)
        tiles, chunks, rows, mpad, S, sps, units, grid, smem = (int(v) for v in out)
        T = -(-K // 256)                                         # the last stage may be half
        assert tiles == -(-N // 128) and chunks == -(-M // 128) and chunks * rows >= M
        assert rows <= 128 and mpad % 16 == 0 and rows <= mpad <= 128
        assert S * sps >= T and (S - 1) * sps < T                  # every split holds a stage
        assert units == tiles * chunks * S and 1 <= grid <= min(units, 148)
        assert smem <= 227 * 1024
    assert W.lib().w4a16_plan(W.PATH_BS, 1, 1, 256, 512, 0, 148, out.ctypes.data, 9) == W.ERR_ARG
    assert W.lib().w4a16_plan(W.PATH_TC, 3, 1, 256, 512, 0, 148, out.ctypes.data, 9) == W.ERR_ARG
