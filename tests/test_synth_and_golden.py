"""The seeded generator and the hand-derived golden examples (CPU only)."""

from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np

import oracle
from oracle import formats
import synth
from exact import bf16_bits_of, e4m3_value, pow2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_splitmix64_published_vector():
    d = _load("splitmix64_seed1234567.json")
    idx = np.arange(len(d["outputs"]), dtype=np.uint64)
    with np.errstate(over="ignore"):
        got = synth.mix64(np.uint64(d["state"]) + (idx + np.uint64(1)) * synth.GAMMA)
    assert [int(v) for v in got] == d["outputs"]


def test_generator_is_counter_based_and_deterministic():
    a = synth.int4_weights(3, 40, 256)
    b = synth.int4_weights(3, 40, 256, rows=[5, 17, 39])
    assert np.array_equal(a[[5, 17, 39]], b)
    assert np.array_equal(a, synth.int4_weights(3, 40, 256))
    assert not np.array_equal(a, synth.int4_weights(4, 40, 256))
    s = synth.int4_scales(3, 40, 256)
    assert np.array_equal(s[[7]], synth.int4_scales(3, 40, 256, rows=[7]))


def test_generator_distributions():
    q = synth.int4_weights(1, 256, 4096)
    assert q.min() == -8 and q.max() == 7
    counts = np.bincount((q.astype(np.int64) + 8).ravel(), minlength=16)
    assert np.all(np.abs(counts / counts.mean() - 1) < 0.02)
    z = synth.normals(5, synth.T_X, np.arange(200000, dtype=np.uint64))
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
    s = formats.bf16_to_f64(synth.int4_scales(2, 512, 5120))
    ls = np.log(s / 0.01)
    assert abs(ls.mean()) < 0.01 and abs(ls.std() - 0.25) < 0.01
    s8 = formats.e4m3_to_f64(synth.nvfp4_scales(6, 512, 1024))
    assert np.all(np.isfinite(s8)) and s8.max() <= 448
    assert abs(s8.mean() - 0.05 * np.sqrt(2 / np.pi)) < 0.002


def test_storage_rounding_of_the_generator_is_rne():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(size=3000), rng.normal(size=500) * 1e-39, [0.0, 1.0, -2.5]])
    bits = synth.to_bf16_bits(v)
    for x, b in zip(v, bits):
        assert int(b) == bf16_bits_of(Fraction(float(x)), negative_zero=np.signbit(x) and x == 0)
    w = np.abs(rng.normal(size=3000)) * 0.05
    w = np.concatenate([w, [0.0, 1e-4, 2.0 ** -10, 2.0 ** -6 * 0.99, 500.0, 448.0, 464.0]])
    enc = synth.to_e4m3_bytes(w)
    finite = [b for b in range(0x7F)]
    for x, b in zip(w, enc):
        # nearest finite E4M3 (ties to even mantissa), saturating at 448
        xr = Fraction(float(x))
        best = min(finite, key=lambda c: (abs(e4m3_value(c) - xr), c & 1))
        if xr > 448:
            best = 0x7E
        assert int(b) == best, (x, hex(int(b)), hex(best))


def test_int4_golden_example_oracle():
    d = _load("int4_worked_example.json")
    k = np.arange(128)
    q = np.stack([(k % 16) - 8, 7 - (k % 16)]).astype(np.int8)
    s = np.array(d["inputs"]["scale_bits"], dtype=np.uint16)
    w = oracle.dequant_int4_g128(q, s)
    want = [int(h, 16) for h in d["expected"]["w_row0_hex_k0_to_15"]]
    assert [int(v) for v in w[0, :16]] == want
    x = np.zeros((1, 128), dtype=np.uint16)
    x[0, :16] = 0x3F80
    assert list(oracle.gemm_ref(x, w)[0]) == d["expected"]["y"]


def test_nvfp4_golden_example_oracle():
    d = _load("nvfp4_worked_example.json")
    c = np.tile(np.arange(16, dtype=np.uint8), (2, 1))
    s8 = np.array(d["inputs"]["scale_e4m3"], dtype=np.uint8)
    w = oracle.dequant_nvfp4(c, s8, d["inputs"]["global_scale"])
    assert [int(v) for v in w[0]] == [int(h, 16) for h in d["expected"]["w_row0_hex_k0_to_15"]]
    x = np.zeros((1, 16), dtype=np.uint16)
    x[0, :8] = 0x3F80
    assert list(oracle.gemm_ref(x, w)[0]) == d["expected"]["y"]


def test_edge_value_problems_reach_the_corners():
    # the edge-value inputs of the GPU parity tests contain what they claim
    p = synth.adversarial_problem("int4", 1, 6, 64, 2048, "extreme")
    s = p["scales"]
    e = (s >> 7) & 0xFF
    assert ((s & 0x8000) != 0).any() and ((s & 0x8000) == 0).any()        # both signs
    assert ((e == 0) & ((s & 0x7F) != 0)).any()                            # subnormal
    assert ((s & 0x7FFF) == 0).any()                                       # zero
    assert (e >= 127 + 90).any() and ((e >= 1) & (e <= 27)).any()          # huge and tiny
    q = p["codes"].reshape(64, -1, 128)
    zero_groups = (q == 0).all(axis=2)
    assert zero_groups.any() and (~zero_groups).any()
    n = synth.adversarial_problem("nvfp4", 2, 3, 32, 1024, "extreme")
    b = n["scales"]
    assert ((b & 0x78) == 0).any() and (b & 0x80).any() and ((b & 0x7F) != 0x7F).all()
    w = synth.adversarial_problem("int4", 3, 3, 16, 1024, "wide")
    xv = oracle.bf16_to_f64(w["x"])
    nz = np.abs(xv[1][xv[1] != 0])
    assert np.log2(nz.max() / nz.min()) > 30                               # a row spans > 2^30
    assert (xv[2] == 0).mean() > 0.9 and np.abs(xv[2]).max() > 2 ** 15
