"""Pins for the fp64 oracle: decoders, rounding, dequantisation and the matmul.

Each check compares the oracle against something other than itself: exact
rational arithmetic built from the formats' bit fields (tests/exact.py),
hand-derived worked examples, closed forms and invariants.  CPU only.
"""

from __future__ import annotations

import random
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import formats
import synth
from exact import (bf16_bits_of, bf16_value, e2m1_value, e4m3_value, fp32_value,
                   E2M1_MAGNITUDES, pow2)

G_NVFP4 = synth.NVFP4_GLOBAL_SCALE          # fp32(1/448)
G_BITS = int(np.float32(G_NVFP4).view(np.uint32))


# ---------------------------------------------------------------- decoders


def test_bf16_decoder_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = formats.bf16_to_f64(bits)
    for b in range(65536):
        ref = bf16_value(b)
        if ref == "nan":
            assert np.isnan(got[b])
        elif ref == "+inf":
            assert got[b] == np.inf
        elif ref == "-inf":
            assert got[b] == -np.inf
        else:
            assert Fraction(got[b]) == ref, hex(b)


def test_e4m3_decoder_exhaustive():
    got = formats.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    for b in range(256):
        ref = e4m3_value(b)
        if ref == "nan":
            assert np.isnan(got[b]), hex(b)
        else:
            assert Fraction(got[b]) == ref, hex(b)
    # landmarks of the OCP definition
    assert got[0x38] == 1.0
    assert got[0x7E] == 448.0
    assert got[0x01] == 2.0 ** -9
    assert got[0x08] == 2.0 ** -6
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0xFE] == -448.0


def test_e2m1_decoder_table():
    got = formats.e2m1_to_f64(np.arange(16, dtype=np.uint8))
    listed = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for c in range(16):
        want = listed[c & 7] * (-1 if c & 8 else 1)
        assert got[c] == want
        assert Fraction(got[c]) == e2m1_value(c)
    assert np.signbit(got[8])                      # code 0x8 is -0
    # field decode agrees with the listed magnitudes
    for c in range(8):
        e, m = (c >> 1) & 3, c & 1
        v = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * pow2(e - 1)
        assert v == E2M1_MAGNITUDES[c]


# ---------------------------------------------------------------- rounding onto BF16


def _random_bf16(rng):
    e = rng.randint(1, 254)
    return (rng.randint(0, 1) << 15) | (e << 7) | rng.randint(0, 127)


def test_rne_bf16_against_exact_rationals():
    rng = random.Random(1234)
    vals = []
    # exact products of the kinds the method forms, plus ties and subnormals
    for _ in range(3000):
        q = rng.randint(-8, 7)
        s = _random_bf16(rng)
        vals.append(q * bf16_value(s))
    for _ in range(2000):
        c = rng.randint(0, 15)
        b = rng.randint(0, 0x7E)
        g = fp32_value(rng.randint(0x30000000, 0x42000000))
        vals.append(e2m1_value(c) * e4m3_value(b) * g)
    # exact midpoints between adjacent BF16 values (ties), subnormal to large
    for b in list(range(0, 0x0100, 7)) + list(range(0x0100, 0x7F7F, 97)):
        lo, hi = bf16_value(b), bf16_value(b + 1)
        vals.append((lo + hi) / 2)
        vals.append(-(lo + hi) / 2)
    x = np.array([float(v) for v in vals], dtype=np.float64)
    assert all(Fraction(float(v)) == v for v in vals)  # binary64 holds every case exactly
    got = formats.f64_to_bf16_rne(x)
    for v, g in zip(vals, got):
        assert int(g) == bf16_bits_of(v), (v, hex(int(g)), hex(bf16_bits_of(v)))


def test_worked_examples_hand_derived():
    # s = BF16 0x3C24 = 1.28125 * 2**-7 = 0.010009765625.
    s = np.array([[0x3C24]], dtype=np.uint16)
    assert formats.bf16_to_f64(s)[0, 0] == 0.010009765625
    # q = 7: 7 s = 0.070068359375 = 143.5 * 2**-11 sits exactly between the BF16
    # neighbours 143 * 2**-11 (0x3D8F) and 144 * 2**-11 (0x3D90); ties go to the
    # even mantissa, 0x3D90 = 0.0703125 (truncation would give 0x3D8F).
    q = np.full((1, 128), 7, dtype=np.int8)
    w = oracle.dequant_int4_g128(q, s)
    assert int(w[0, 0]) == 0x3D90
    # q = -8: -8 s = -0.080078125 is exact in BF16: 0xBDA4.
    w = oracle.dequant_int4_g128(np.full((1, 128), -8, dtype=np.int8), s)
    assert int(w[0, 0]) == 0xBDA4
    # NVFP4: code 7 (6.0) x E4M3 0x38 (1.0) x fp32(1/448): 6/448 = 1.7142857 * 2**-7
    # -> 8-bit significand 219.43/128 -> 219 -> 0x3C5B = 0.01336669921875.
    c = np.full((1, 16), 7, dtype=np.uint8)
    w = oracle.dequant_nvfp4(c, np.array([[0x38]], dtype=np.uint8), G_NVFP4)
    assert int(w[0, 0]) == 0x3C5B
    assert formats.bf16_to_f64(w)[0, 0] == 0.01336669921875
    # code 3 (1.5) x 0x30 (0.5) x g = 0.75/448 -> 0.00167083740234375
    c = np.full((1, 16), 3, dtype=np.uint8)
    w = oracle.dequant_nvfp4(c, np.array([[0x30]], dtype=np.uint8), G_NVFP4)
    assert formats.bf16_to_f64(w)[0, 0] == 0.00167083740234375


# ---------------------------------------------------------------- dequantisation


def _stratified_bf16_scales():
    """Every sign/exponent with 16 mantissas, plus all mantissas of 3 binades."""
    out = set()
    for sign in (0, 1):
        for e in range(0, 255):                  # finite exponents incl. subnormal
            for m in range(0, 128, 8):
                out.add((sign << 15) | (e << 7) | m)
            out.add((sign << 15) | (e << 7) | 127)
    for e in (1, 120, 254):
        for m in range(128):
            out.add((e << 7) | m)
    return sorted(out)


def test_dequant_int4_all_codes_stratified_scales():
    scales = _stratified_bf16_scales()
    q = np.tile(np.repeat(np.arange(-8, 8, dtype=np.int8), 8), (len(scales), 1))  # K = 128
    s = np.array(scales, dtype=np.uint16)[:, None]
    w = oracle.dequant_int4_g128(q, s)
    for i, sb in enumerate(scales):
        sv = bf16_value(sb)
        for j in range(0, 128, 8):
            qv = int(q[i, j])
            prod = qv * sv
            neg_zero = (prod == 0) and ((qv < 0) != (sb >= 0x8000)) and qv != 0
            want = bf16_bits_of(prod, negative_zero=neg_zero)
            got = int(w[i, j])
            if prod == 0:
                assert got & 0x7FFF == 0
            else:
                assert got == want, (qv, hex(sb), hex(got), hex(want))


@pytest.mark.parametrize("g_bits", [G_BITS, 0x3F800000, 0x3DCCCCCD, 0x3B449BA6, 0x4B7FFFFF])
def test_dequant_nvfp4_all_code_scale_pairs(g_bits):
    g = float(np.array([g_bits], dtype=np.uint32).view(np.float32)[0])
    finite = [b for b in range(256) if e4m3_value(b) != "nan"]
    codes = np.tile(np.arange(16, dtype=np.uint8), (len(finite), 1))     # K = 16
    s8 = np.array(finite, dtype=np.uint8)[:, None]
    w = oracle.dequant_nvfp4(codes, s8, g)
    gv = fp32_value(g_bits)
    for i, b in enumerate(finite):
        for c in range(16):
            prod = e2m1_value(c) * e4m3_value(b) * gv
            got = int(w[i, c])
            if prod == 0:
                assert got & 0x7FFF == 0
            else:
                assert got == bf16_bits_of(prod), (c, hex(b), hex(got))


def test_dequant_group_index_is_k_div_group():
    # one distinct power-of-two scale per group: the group a k belongs to is
    # read back from the exponent of W_deq when q = 1
    N, K = 3, 512
    q = np.ones((N, K), dtype=np.int8)
    s = np.zeros((N, K // 128), dtype=np.uint16)
    for n in range(N):
        for g in range(K // 128):
            s[n, g] = (127 + 4 * g + n) << 7     # 2**(4g+n)
    w = formats.bf16_to_f64(oracle.dequant_int4_g128(q, s))
    for n in range(N):
        for k in range(K):
            assert w[n, k] == 2.0 ** (4 * (k // 128) + n)
    c = np.full((2, 64), 2, dtype=np.uint8)        # e2m1 code 2 = 1.0
    s8 = np.zeros((2, 4), dtype=np.uint8)
    for n in range(2):
        for g in range(4):
            s8[n, g] = (7 + g + 2 * n) << 3       # 2**(g+2n)
    w = formats.bf16_to_f64(oracle.dequant_nvfp4(c, s8, 1.0))
    for n in range(2):
        for k in range(64):
            assert w[n, k] == 2.0 ** ((k // 16) + 2 * n)


def test_dequant_rejects_out_of_contract_inputs():
    with pytest.raises(ValueError):
        oracle.dequant_int4_g128(np.full((1, 128), 8, dtype=np.int8), np.zeros((1, 1), np.uint16))
    with pytest.raises(ValueError):
        oracle.dequant_int4_g128(np.zeros((1, 100), dtype=np.int8), np.zeros((1, 1), np.uint16))
    with pytest.raises(ValueError):
        oracle.dequant_nvfp4(np.zeros((1, 16), np.uint8), np.array([[0x7F]], np.uint8), 1.0)


# ---------------------------------------------------------------- the matmul


def _exact_y(x_bits, w_bits):
    M, K = x_bits.shape
    N = w_bits.shape[0]
    xs = [[bf16_value(int(b)) for b in row] for row in x_bits]
    ws = [[bf16_value(int(b)) for b in row] for row in w_bits]
    return [[sum(xs[m][k] * ws[n][k] for k in range(K)) for n in range(N)] for m in range(M)]


@pytest.mark.parametrize("fmt,M,N,K,seed", [("int4", 1, 4, 128, 11), ("int4", 3, 2, 256, 12),
                                             ("nvfp4", 2, 3, 128, 13), ("nvfp4", 1, 4, 256, 14)])
def test_gemm_brute_force_exact(fmt, M, N, K, seed):
    p = synth.problem(fmt, seed, M, N, K)
    w = (oracle.dequant_int4_g128(p["codes"], p["scales"]) if fmt == "int4"
         else oracle.dequant_nvfp4(p["codes"], p["scales"], p["g"]))
    y = oracle.gemm_ref(p["x"], w)
    bound = oracle.abs_bound(p["x"], w)
    ex = _exact_y(p["x"], w)
    for m in range(M):
        for n in range(N):
            # binary64 accumulation of K exact products: error <= K * 2**-53 * bound
            assert abs(Fraction(y[m, n]) - ex[m][n]) <= Fraction(K) * pow2(-52) * Fraction(bound[m, n])
            assert abs(y[m, n]) <= bound[m, n] * (1 + 1e-12)


def _exact_abs_bound(x_bits, w_bits):
    """sum_k |x[m][k] * W_deq[n][k]| in exact rationals, by loops over k."""
    M, K = x_bits.shape
    N = w_bits.shape[0]
    xs = [[abs(bf16_value(int(b))) for b in row] for row in x_bits]
    ws = [[abs(bf16_value(int(b))) for b in row] for row in w_bits]
    return [[sum(xs[m][k] * ws[n][k] for k in range(K)) for n in range(N)] for m in range(M)]


def _bound_pins(bound_fn):
    """Checks of a tolerance-scale function against what fixes sum_k |W x|;
    returns the names of the checks it fails."""
    fails = []
    # exact rationals on seeded brute-force shapes of both formats
    for fmt, M, N, K, seed in (("int4", 2, 3, 256, 15), ("nvfp4", 3, 2, 128, 16)):
        p = synth.problem(fmt, seed, M, N, K)
        w = (oracle.dequant_int4_g128(p["codes"], p["scales"]) if fmt == "int4"
             else oracle.dequant_nvfp4(p["codes"], p["scales"], p["g"]))
        b = bound_fn(p["x"], w)
        ex = _exact_abs_bound(p["x"], w)
        # K non-negative exact products summed in binary64: relative error <= K * 2**-53
        if any(abs(Fraction(b[m, n]) - ex[m][n]) > Fraction(K) * pow2(-53) * ex[m][n]
               for m in range(M) for n in range(N)):
            fails.append("exact")
    # closed form: x = (1, -1, 1, -1, ...) and W_deq = 1 everywhere cancel to
    # y = 0 while the bound counts every term: K
    K = 256
    x = np.tile(np.array([0x3F80, 0xBF80], np.uint16), (1, K // 2))
    w = np.full((2, K), 0x3F80, np.uint16)
    if not np.all(bound_fn(x, w) == K):
        fails.append("cancelling signs")
    # one term: |x_k| * |W_k| for a negative x and a negative weight
    x1 = np.zeros((1, K), np.uint16)
    x1[0, 7] = 0xC040                        # -3
    w1 = np.zeros((1, K), np.uint16)
    w1[0, 7] = 0xBF00                        # -0.5
    w1[0, 8] = 0x4000                        # 2, paired with x = 0: contributes 0
    if bound_fn(x1, w1)[0, 0] != 1.5:
        fails.append("one term")
    return fails


def test_abs_bound_pinned():
    assert _bound_pins(oracle.abs_bound) == []


def test_abs_bound_pins_catch_planted_mistakes():
    def abs_outside(x, w):         # |sum_k x w| instead of sum_k |x w|
        return np.abs(oracle.gemm_ref(x, w))

    def abs_of_x_only(x, w):       # forgets the weights' signs
        return np.abs(formats.bf16_to_f64(x)) @ formats.bf16_to_f64(w).T

    def abs_of_w_only(x, w):       # forgets the activations' signs
        return formats.bf16_to_f64(x) @ np.abs(formats.bf16_to_f64(w)).T

    def dropped_term(x, w):        # drops the last k
        return np.abs(formats.bf16_to_f64(x))[:, :-1] @ np.abs(formats.bf16_to_f64(w))[:, :-1].T

    for mutant in (abs_outside, abs_of_x_only, abs_of_w_only, dropped_term):
        assert _bound_pins(mutant) != [], mutant.__name__
    assert "cancelling signs" in _bound_pins(abs_outside)


def _int4_case(seed=21, M=4, N=40, K=384):
    p = synth.problem("int4", seed, M, N, K)
    return p, oracle.dequant_int4_g128(p["codes"], p["scales"])


def test_invariant_zero_scales_give_zero():
    p, _ = _int4_case()
    w = oracle.dequant_int4_g128(p["codes"], np.zeros_like(p["scales"]))
    assert np.all(oracle.gemm_ref(p["x"], w) == 0)
    c = synth.nvfp4_codes(3, 8, 64)
    w = oracle.dequant_nvfp4(c, np.zeros((8, 4), np.uint8), G_NVFP4)
    assert np.all(formats.bf16_to_f64(w) == 0)


def test_invariant_one_hot_selects_a_dequantised_column():
    p, w = _int4_case()
    K = p["K"]
    for k in (0, 1, 127, 128, 200, K - 1):
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = 0x3F80                               # 1.0
        y = oracle.gemm_ref(x, w)
        assert np.array_equal(y[0], formats.bf16_to_f64(w[:, k]))


def test_invariant_power_of_two_scaling_is_exact():
    p, w = _int4_case()
    x2 = (p["x"].astype(np.int32) + (1 << 7)).astype(np.uint16)     # exponent + 1: 2x
    nz = (p["x"] & 0x7F80) != 0
    x2 = np.where(nz, x2, p["x"])
    assert np.array_equal(oracle.gemm_ref(x2, w), 2 * oracle.gemm_ref(p["x"], w))


def test_invariant_linearity_and_row_independence():
    p, w = _int4_case()
    x1 = formats.bf16_to_f64(p["x"])
    x2 = formats.bf16_to_f64(synth.activations(99, p["M"], p["K"]))
    # a and b chosen so that a*x1 + b*x2 stays exact enough: compare in fp64
    lhs = (0.5 * x1 + 0.25 * x2) @ formats.bf16_to_f64(w).T
    rhs = 0.5 * oracle.gemm_ref(p["x"], w) + 0.25 * oracle.gemm_ref(synth.activations(99, p["M"], p["K"]), w)
    bound = oracle.abs_bound(p["x"], w) + oracle.abs_bound(synth.activations(99, p["M"], p["K"]), w)
    assert np.all(np.abs(lhs - rhs) <= 1e-12 * bound + 1e-300)
    y = oracle.gemm_ref(p["x"], w)
    for m in range(p["M"]):
        assert np.array_equal(oracle.gemm_ref(p["x"][m:m + 1], w)[0], y[m])


def test_invariant_column_permutation():
    p, w = _int4_case()
    perm = np.random.default_rng(5).permutation(p["N"])
    wp = oracle.dequant_int4_g128(p["codes"][perm], p["scales"][perm])
    assert np.array_equal(oracle.gemm_ref(p["x"], wp), oracle.gemm_ref(p["x"], w)[:, perm])


def test_tolerance_helper():
    y_ref = np.array([[1.0, -2.0]])
    bound = np.array([[128.0, 0.0]])
    ok, ex = oracle.within_tolerance(np.array([[2.0, -2.0005]]), y_ref, bound)
    assert ok.all()
    ok, ex = oracle.within_tolerance(np.array([[2.01, -2.002]]), y_ref, bound)
    assert not ok.any()


# ---------------------------------------------------------------- planted mistakes


def _pin_suite(dequant_int4, gemm):
    """A compact re-run of the pins above against a (possibly mutated) oracle."""
    fails = []
    s = np.array([[0x3C24]], dtype=np.uint16)
    if int(dequant_int4(np.full((1, 128), 7, np.int8), s)[0, 0]) != 0x3D90:
        fails.append("tie")
    if int(dequant_int4(np.full((1, 128), -8, np.int8), s)[0, 0]) != 0xBDA4:
        fails.append("sign")
    N, K = 2, 256
    q = np.ones((N, K), dtype=np.int8)
    sc = np.array([[0x3F80, 0x4000], [0x4080, 0x4100]], dtype=np.uint16)   # 1, 2, 4, 8
    w = formats.bf16_to_f64(dequant_int4(q, sc))
    if not (np.all(w[0, :128] == 1) and np.all(w[0, 128:] == 2) and np.all(w[1, :128] == 4)
            and np.all(w[1, 128:] == 8)):
        fails.append("group index")
    p = synth.problem("int4", 31, 2, 3, 256)
    wd = oracle.dequant_int4_g128(p["codes"], p["scales"])
    y = gemm(p["x"], wd)
    ex = _exact_y(p["x"], wd)
    if any(abs(Fraction(y[m, n]) - ex[m][n]) > Fraction(1, 1 << 30) for m in range(2) for n in range(3)):
        fails.append("matmul")
    return fails


def test_pins_catch_planted_mistakes():
    assert _pin_suite(oracle.dequant_int4_g128, oracle.gemm_ref) == []

    def truncating(q, s):          # rounds toward zero instead of to nearest even
        v = q.astype(np.float64) * np.repeat(formats.bf16_to_f64(s), 128, axis=1)
        return (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)

    def wrong_group(q, s):         # scale index k // 64 instead of k // 128
        idx = np.minimum(np.arange(q.shape[1]) // 64, s.shape[1] - 1)
        v = q.astype(np.float64) * formats.bf16_to_f64(s)[:, idx]
        return formats.f64_to_bf16_rne(v)

    def offset_sign(q, s):         # uses the stored offset-binary code q + 8 as the value
        v = (q.astype(np.float64) + 8) * np.repeat(formats.bf16_to_f64(s), 128, axis=1)
        return formats.f64_to_bf16_rne(v)

    def transposed(x, w):          # transposed operand / wrong axis of the sum
        xf, wf = formats.bf16_to_f64(x), formats.bf16_to_f64(w)
        return (xf[:, ::-1] @ wf.T)

    def dropped_term(x, w):        # drops the last product of every dot product
        xf, wf = formats.bf16_to_f64(x), formats.bf16_to_f64(w)
        return xf[:, :-1] @ wf[:, :-1].T

    assert "tie" in _pin_suite(truncating, oracle.gemm_ref)
    assert "group index" in _pin_suite(wrong_group, oracle.gemm_ref)
    assert "sign" in _pin_suite(offset_sign, oracle.gemm_ref)
    assert "matmul" in _pin_suite(oracle.dequant_int4_g128, transposed)
    assert "matmul" in _pin_suite(oracle.dequant_int4_g128, dropped_term)


# ---------------------------------------------------------------- fused gate/up + SiLU


def test_silu_closed_forms():
    import math
    s = oracle.silu(np.array([0.0, 1.0, -1.0, 2.0, 50.0, -50.0, -800.0, 800.0]))
    # sigmoid(1) = e / (1 + e), sigmoid(2) = e^2 / (1 + e^2): textbook values
    assert s[0] == 0.0
    assert abs(s[1] - 0.7310585786300049) <= 1e-16
    assert abs(s[2] - (-0.2689414213699951)) <= 1e-16
    assert abs(s[3] - 2 * math.e ** 2 / (1 + math.e ** 2)) <= 1e-15   # a few ulps
    assert s[4] == 50.0                                  # sigmoid(50) rounds to 1
    assert abs(s[5]) < 1e-19 and s[5] < 0                # -50 * e^-50
    assert s[6] == 0.0 and np.signbit(s[6])              # the limit, no NaN from inf / inf
    assert s[7] == 800.0
    # SiLU(z) - SiLU(-z) = z: sigmoid(z) + sigmoid(-z) = 1
    z = np.linspace(-30, 30, 121)
    assert np.allclose(oracle.silu(z) - oracle.silu(-z), z, rtol=0, atol=1e-13)


def _silu_brute(x_bits, w_bits):
    """h by pure-Python loops from the formats' bit fields and math.exp."""
    import math
    M, K = x_bits.shape
    N = w_bits.shape[0]
    I = N // 2
    ex = _exact_y(x_bits, w_bits)
    out = []
    for m in range(M):
        row = []
        for i in range(I):
            g, u = float(ex[m][i]), float(ex[m][I + i])
            row.append(g / (1.0 + math.exp(-g)) * u if g > -700 else 0.0 * u)
        out.append(row)
    return out


@pytest.mark.parametrize("fmt,M,I,K,seed", [("int4", 2, 3, 128, 31), ("nvfp4", 3, 2, 256, 32)])
def test_gate_up_silu_brute_force(fmt, M, I, K, seed):
    p = synth.problem(fmt, seed, M, 2 * I, K)
    w = (oracle.dequant_int4_g128(p["codes"], p["scales"]) if fmt == "int4"
         else oracle.dequant_nvfp4(p["codes"], p["scales"], p["g"]))
    h, gate, up = oracle.gate_up_silu_ref(p["x"], w)
    assert h.shape == (M, I) and gate.shape == (M, I) and up.shape == (M, I)
    ref = _silu_brute(p["x"], w)
    for m in range(M):
        for i in range(I):
            assert abs(h[m, i] - ref[m][i]) <= 1e-12 * max(1.0, abs(ref[m][i]))


def test_gate_up_silu_layout_and_tolerance():
    p = synth.problem("int4", 33, 4, 2 * 24, 384)
    w = oracle.dequant_int4_g128(p["codes"], p["scales"])
    h, gate, up = oracle.gate_up_silu_ref(p["x"], w)
    y = oracle.gemm_ref(p["x"], w)
    # gate rows first, up rows second (not interleaved, not swapped)
    assert np.array_equal(gate, y[:, :24]) and np.array_equal(up, y[:, 24:])
    allowed = oracle.gate_up_silu_allowed(p["x"], w, gate, up)
    assert np.all(allowed > 0)
    # the exact value and its BF16 rounding pass
    hb = formats.bf16_to_f64(formats.f64_to_bf16_rne(h))
    assert np.all(np.abs(hb - h) <= allowed)
    # plausible mistakes fail: halves swapped, SiLU on the wrong half, SiLU left out
    for wrong in (oracle.silu(up) * gate, gate * up, oracle.silu(gate) * gate):
        assert np.any(np.abs(wrong - h) > allowed)


# ---------------------------------------------------------------- FP8-E4M3 weights (W8A16)


@pytest.mark.parametrize("g_bits", [0x3B124925, 0x3F800000, 0x3DCCCCCD, 0x0DA24260])
def test_dequant_fp8_every_code(g_bits):
    # every finite E4M3 byte times the fp32 scale, against exact rationals
    g = float(np.array([g_bits], dtype=np.uint32).view(np.float32)[0])
    finite = [b for b in range(256) if e4m3_value(b) != "nan"]
    codes = np.array(finite, dtype=np.uint8)[None, :]
    w = oracle.dequant_fp8_e4m3(codes, g)
    gv = fp32_value(g_bits)
    for i, b in enumerate(finite):
        prod = e4m3_value(b) * gv
        got = int(w[0, i])
        if prod == 0:
            assert got & 0x7FFF == 0 and (got >> 15) == (b >> 7), hex(b)   # signed zeros kept
        else:
            assert got == bf16_bits_of(prod), (hex(b), hex(got))


def test_dequant_fp8_rejects_nan_and_is_elementwise():
    with pytest.raises(ValueError):
        oracle.dequant_fp8_e4m3(np.array([[0x7F]], np.uint8), 1.0)
    with pytest.raises(ValueError):
        oracle.dequant_fp8_e4m3(np.array([[0xFF]], np.uint8), 1.0)
    # no grouping: permuting the codes permutes the weights
    c = synth.fp8_weights(5, 3, 128)
    perm = np.random.default_rng(0).permutation(128)
    g = synth.FP8_GLOBAL_SCALE
    assert np.array_equal(oracle.dequant_fp8_e4m3(c[:, perm], g), oracle.dequant_fp8_e4m3(c, g)[:, perm])


def test_fp8_gemm_brute_force_exact():
    p = synth.problem("fp8", 15, 2, 3, 128)
    w = oracle.dequant_fp8_e4m3(p["codes"], p["g"])
    y = oracle.gemm_ref(p["x"], w)
    bound = oracle.abs_bound(p["x"], w)
    ex = _exact_y(p["x"], w)
    for m in range(2):
        for n in range(3):
            assert abs(Fraction(y[m, n]) - ex[m][n]) <= Fraction(128) * pow2(-52) * Fraction(bound[m, n])


def test_fp8_draws_follow_the_recipe():
    c = synth.fp8_weights(7, 64, 1024)
    v = formats.e4m3_to_f64(c)
    assert np.all(np.isfinite(v)) and np.abs(v).max() <= 448
    z = v / 64.0                                   # back to the N(0, 1) scale, up to rounding
    assert abs(z.mean()) < 0.02 and abs(z.std() - 1.0) < 0.03
    # the sign comes from the draw: about half negative
    assert 0.45 < np.mean(c >= 0x80) < 0.55


# ---------------------------------------------------------------- W4A4 NVFP4 groundwork (activation quantiser)


def test_e2m1_rounding_table():
    # the E2M1 grid 0, 0.5, 1, 1.5, 2, 3, 4, 6; ties go to the code with mantissa bit 0
    cases = [(0.0, 0), (0.2, 0), (0.25, 0), (0.3, 1), (0.75, 2), (1.25, 2), (1.3, 3), (1.75, 4),
             (2.5, 4), (2.6, 5), (3.5, 6), (5.0, 6), (5.1, 7), (6.0, 7), (7.5, 7), (1e30, 7)]
    v = np.array([c[0] for c in cases])
    assert list(formats.f64_to_e2m1_rne(v)) == [c[1] for c in cases]
    assert list(formats.f64_to_e2m1_rne(-v)) == [c[1] | 8 for c in cases]       # sign bit, -0 too
    # every code decodes back to itself
    codes = np.arange(16, dtype=np.uint8)
    back = formats.f64_to_e2m1_rne(formats.e2m1_to_f64(codes))
    assert np.array_equal(back, codes)


def test_e4m3_encoder_round_trip_ties_and_saturation():
    finite = np.array([b for b in range(0x7F)], dtype=np.uint8)           # non-negative, no NaN
    vals = formats.e4m3_to_f64(finite)
    assert np.array_equal(formats.f64_to_e4m3_rne(vals), finite)
    # midpoints between neighbours: ties to the even code (mantissa LSB 0)
    mids = (vals[:-1] + vals[1:]) / 2
    want = np.where(finite[:-1] % 2 == 0, finite[:-1], finite[1:])
    assert np.array_equal(formats.f64_to_e4m3_rne(mids), want)
    assert formats.f64_to_e4m3_rne(np.array([449.0, 1e9]))[0] == 0x7E           # saturates at 448
    with pytest.raises(ValueError):
        formats.f64_to_e4m3_rne(np.array([-1.0]))


def test_w4a4_quantiser_reproduces_representable_blocks():
    # rows built as e2m1 * e4m3 * g_x with the block's largest magnitude 6:
    # the quantiser must return exactly those codes and scales
    rng = np.random.default_rng(5)
    g = 2.0 ** -9                  # a power of two keeps every product exact in BF16
    M, K = 3, 64
    codes = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    codes[:, ::16] = 7                                                     # each block reaches +6
    s8 = rng.integers(0x20, 0x60, size=(M, K // 16)).astype(np.uint8)
    x = formats.e2m1_to_f64(codes) * np.repeat(formats.e4m3_to_f64(s8), 16, axis=1) * g
    x_bits = formats.f64_to_bf16_rne(x)
    assert np.array_equal(formats.bf16_to_f64(x_bits), x)                  # exactly representable
    q, s = oracle.w4a4.quantize_activations(x_bits, g)
    assert np.array_equal(s, s8)
    zero = formats.e2m1_to_f64(codes) == 0
    assert np.array_equal(q[~zero], codes[~zero])                           # +-0 may differ in sign only


def test_w4a4_quantiser_zero_blocks_scale_and_error_bound():
    p = synth.problem("int4", 41, 4, 1, 256)
    x_bits = p["x"].copy()
    x_bits[1, 32:48] = 0                                                    # one all-zero block
    g = oracle.w4a4.activation_global_scale(x_bits)
    q, s = oracle.w4a4.quantize_activations(x_bits, g)
    assert s[1, 2] == 0 and np.all(formats.e2m1_to_f64(q[1, 32:48]) == 0)
    x = formats.bf16_to_f64(x_bits)
    xh = oracle.w4a4.dequant_activations(q, s, g)
    amax = np.repeat(np.abs(x).reshape(4, 16, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(xh - x) <= 0.25 * amax + 1e-30)                   # E2M1 spacing + scale rounding
    # the block's largest element maps to the top of the grid (|code| 6, or 4 after a scale round-up)
    top = np.abs(formats.e2m1_to_f64(q)).reshape(4, 16, 16).max(axis=2)
    assert np.all(np.isin(top[s > 0], [4.0, 6.0]))
    # the tensor's largest magnitude sets g_x: its block scale is 448 (or just below)
    assert formats.e4m3_to_f64(s).max() >= 416


def test_w4a4_gemm_brute_force_exact():
    from exact import e2m1_value, e4m3_value, fp32_value
    M, N, K = 2, 3, 32
    px = synth.problem("int4", 42, M, 1, K)
    g_x = oracle.w4a4.activation_global_scale(px["x"])
    xq, xs = oracle.w4a4.quantize_activations(px["x"], g_x)
    pw = synth.problem("nvfp4", 43, 1, N, K)
    y = oracle.w4a4.gemm_w4a4_ref(xq, xs, g_x, pw["codes"], pw["scales"], pw["g"])
    gx = fp32_value(int(np.array([g_x], np.float32).view(np.uint32)[0]))
    gw = fp32_value(int(np.array([pw["g"]], np.float32).view(np.uint32)[0]))
    for m in range(M):
        for n in range(N):
            ex = sum(e2m1_value(int(xq[m, k])) * e4m3_value(int(xs[m, k // 16])) * gx *
                     e2m1_value(int(pw["codes"][n, k])) * e4m3_value(int(pw["scales"][n, k // 16])) * gw
                     for k in range(K))
            # exact block-scaled sum, then two roundings by the fp32 scales
            assert abs(Fraction(y[m, n]) - ex) <= pow2(-51) * abs(ex)
