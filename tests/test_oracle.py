"""Pins of the CPU oracle against facts fixed by the mathematics, not by the oracle itself.

Each test checks the oracle against something independent of its own code:
a textbook matrix, scipy's Hadamard routine, hand-derived closed forms
(tests/golden/closed_forms.json), exact rational arithmetic, brute-force
integer loops, or an invariant of the method (orthogonality, the rotation
invariance X R (W R)^T = X W^T, equivariance, symmetry). A plausible slip in
the oracle (a dropped 1/sqrt(g), a transposed Hadamard, a wrong block index, a
wrong tie rule, a per-tensor instead of per-token scale, a missing bias or
scale factor) fails at least one of them.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle
import synth


def _hex(s: str) -> float:
    return float.fromhex(s)


# ---------------------------------------------------------------- rotation


def test_hadamard_g2_is_textbook():
    assert np.array_equal(oracle.hadamard(2), np.array([[1.0, 1.0], [1.0, -1.0]]))


@pytest.mark.parametrize("g", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_recursive_sylvester(g):
    h = np.array([[1.0]])
    while h.shape[0] < g:
        h = np.block([[h, h], [h, -h]])
    assert np.array_equal(oracle.hadamard(g), h)


@pytest.mark.parametrize("g", [2, 4, 16, 128, 256])
def test_hadamard_matches_scipy(g):
    assert np.array_equal(oracle.hadamard(g), scipy.linalg.hadamard(g).astype(np.float64))


@pytest.mark.parametrize("g", [128, 256])
def test_rotation_is_orthonormal(g):
    R = oracle.rotation_matrix(3 * g, g)
    err = np.max(np.abs(R @ R.T - np.eye(3 * g)))
    assert err < 1e-12  # required: 1e-6


@pytest.mark.parametrize("K,g", [(256, 256), (512, 128), (768, 256), (16, 4)])
def test_rotate_equals_block_diagonal_product(K, g):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, K))
    R = np.kron(np.eye(K // g), scipy.linalg.hadamard(g) / math.sqrt(g))
    assert np.allclose(oracle.rotate(x, g), x @ R, rtol=0, atol=1e-12)


@pytest.mark.parametrize("g", [128, 256])
def test_rotation_invariance(g):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((9, 4 * g))
    w = rng.standard_normal((13, 4 * g))
    lhs = oracle.rotate(x, g) @ oracle.rotate(w, g).T
    rhs = x @ w.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


# ---------------------------------------------------------- quantisation


def test_golden_quant_cases(golden):
    for case in golden["quant_cases"]:
        g = case["g"]
        x = np.array([case["x"]], dtype=np.float64)
        rot = oracle.rotate(x, g)
        assert np.array_equal(rot[0], np.array(case["rotated"])), case["name"]
        q, s = oracle.quant_act(x, g)
        assert q.dtype == np.int8
        assert q[0].tolist() == case["codes"], case["name"]
        assert float(s[0]) == _hex(case["scale_hex"]), case["name"]


def test_tie_rule_on_rotated_rows():
    # already-rotated row with absmax 127 -> scale exactly 1
    row = np.array([[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 126.5]])
    q, s = oracle.quantize_per_token(row)
    assert float(s[0]) == 1.0
    assert q[0].tolist() == [127, 2, 4, -2, -4, 0, 2, 0, 126]


@pytest.mark.parametrize("g", [128, 256])
@pytest.mark.parametrize("j,c", [(0, 1.0), (37, -3.0), (255, 0.125), (130, 1e-3)])
def test_spike_row_closed_form(g, j, c):
    K = 2 * g
    x = np.zeros((1, K))
    x[0, j] = c
    q, s = oracle.quant_act(x, g)
    blk = j // g
    expect = np.zeros(K, dtype=np.int64)
    expect[blk * g:(blk + 1) * g] = 127 * int(np.sign(c)) * scipy.linalg.hadamard(g)[j % g]
    assert np.array_equal(q[0].astype(np.int64), expect)
    s_closed = abs(c) / (math.sqrt(g) * 127.0)
    assert abs(float(s[0]) - s_closed) <= 1.2e-7 * s_closed


@pytest.mark.parametrize("g", [128, 256])
@pytest.mark.parametrize("c", [1.0, -0.75, 40.0])
def test_constant_group_closed_form(g, c):
    K = 3 * g
    x = np.zeros((1, K))
    x[0, g:2 * g] = c
    q, s = oracle.quant_act(x, g)
    expect = np.zeros(K, dtype=np.int64)
    expect[g] = 127 * int(np.sign(c))
    assert np.array_equal(q[0].astype(np.int64), expect)
    s_closed = abs(c) * math.sqrt(g) / 127.0
    assert abs(float(s[0]) - s_closed) <= 1.2e-7 * s_closed


def _tiny():
    d = synth.make_workload("tiny")
    return d, oracle.bf16_to_f64(d["x"]), oracle.bf16_to_f64(d["w"])


def test_codes_in_range_and_every_row_hits_127():
    d, x, _ = _tiny()
    q, s = oracle.quant_act(x, d["workload"].g)
    assert q.min() >= -127 and q.max() <= 127
    assert np.all(np.max(np.abs(q.astype(np.int32)), axis=1) == 127)
    assert np.all(s > 0)


def test_scale_is_per_token():
    # two tokens with very different ranges keep their own scales
    _, x, _ = _tiny()
    x2 = np.stack([x[0], 1000.0 * x[0], x[1]])
    q, s = oracle.quant_act(x2, 256)
    assert s[1] == pytest.approx(1000.0 * s[0], rel=1e-6)
    assert np.array_equal(q[0], q[1])
    # each token's codes do not depend on the other tokens in the batch
    q1, s1 = oracle.quant_act(x2[2:], 256)
    assert np.array_equal(q[2], q1[0]) and s[2] == s1[0]


@pytest.mark.parametrize("k", [-6, -1, 3, 9])
def test_scale_equivariance_power_of_two(k):
    _, x, _ = _tiny()
    q0, s0 = oracle.quant_act(x, 256)
    q1, s1 = oracle.quant_act(x * 2.0**k, 256)
    assert np.array_equal(q0, q1)
    assert np.array_equal(s1, (s0.astype(np.float64) * 2.0**k).astype(np.float32))


def test_odd_symmetry():
    _, x, _ = _tiny()
    q0, s0 = oracle.quant_act(x, 256)
    q1, s1 = oracle.quant_act(-x, 256)
    assert np.array_equal(q1, -q0)
    assert np.array_equal(s0, s1)


def test_tensorwise_weight_quant():
    d, _, w = _tiny()
    wq, s_w = oracle.prepare_weight(w, 256)
    wr = scipy.linalg.hadamard(256) / 16.0
    w_rot = w @ wr  # one group: K = g = 256
    assert float(s_w) == float(np.float32(np.max(np.abs(w_rot)) / 127.0))
    assert np.max(np.abs(wq.astype(np.int32))) == 127
    # every code is within half a step of the scaled value (rounding to nearest)
    assert np.max(np.abs(wq - w_rot / np.float64(s_w))) <= 0.5 + 1e-9


# --------------------------------------------------------------- GEMM


def test_gemm_bruteforce_loops_tiny():
    rng = np.random.default_rng(5)
    a = rng.integers(-127, 128, size=(7, 256), dtype=np.int64)
    b = rng.integers(-127, 128, size=(9, 256), dtype=np.int64)
    acc = oracle.gemm_s32(a.astype(np.int8), b.astype(np.int8))
    for m in range(7):
        for n in range(9):
            tot = 0
            for k in range(256):
                tot += int(a[m, k]) * int(b[n, k])
            assert acc[m, n] == tot


def test_gemm_extreme_codes_exact():
    # all +-127 over K = 12288: |acc| = 12288 * 127^2 = 198193152, exact in int32
    K = 12288
    a = np.full((2, K), 127, np.int8)
    a[1] = -127
    b = np.full((3, K), 127, np.int8)
    b[2, ::2] = -127
    acc = oracle.gemm_s32(a, b)
    assert acc[0, 0] == K * 127 * 127
    assert acc[1, 1] == -K * 127 * 127
    assert acc[0, 2] == 0


def test_gemm_matches_integer_matmul_on_tiny_workload():
    d, x, w = _tiny()
    xq, _ = oracle.quant_act(x, 256)
    wq, _ = oracle.prepare_weight(w, 256)
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(oracle.gemm_s32(xq, wq).astype(np.int64), ref)


# --------------------------------------------------- end to end / dequant


def test_golden_linear_case(golden):
    c = golden["linear_case"]
    g = c["g"]
    x = np.array(c["x"])
    w = np.array(c["w"])
    bias = np.array(c["bias"])
    xq, s_x = oracle.quant_act(x, g)
    wq, s_w = oracle.prepare_weight(w, g)
    assert xq.tolist() == c["x_codes"]
    assert [float(v) for v in s_x] == [_hex(h) for h in c["x_scale_hex"]]
    assert wq.tolist() == c["w_codes"]
    assert float(s_w) == _hex(c["w_scale_hex"])
    acc = oracle.gemm_s32(xq, wq)
    assert acc.tolist() == c["acc"]
    y = oracle.linear(x, wq, s_w, g, bias)
    sw = _hex(c["w_scale_hex"])
    for m in range(2):
        for n in range(2):
            expect = c["acc"][m][n] * (_hex(c["x_scale_hex"][m]) * sw) + c["bias"][n]
            assert y[m, n] == expect


def _round_half_even(fr: Fraction) -> int:
    return round(fr)  # Python rounds Fractions half to even


def _exact_linear(x, w, bias, g):
    """Exact rational ConvRot linear for g in {4, 16} (1/sqrt(g) rational)."""
    h2 = [[1, 1], [1, -1]]
    h = [[1]]
    while len(h) < g:  # Kronecker square of the textbook 2x2
        h = [[a * b for a in ra for b in rb] for ra in h for rb in h2]
    inv_sqrt_g = Fraction(1, int(math.isqrt(g)))

    def rot(row):
        out = []
        for b0 in range(0, len(row), g):
            blk = row[b0:b0 + g]
            for k in range(g):
                out.append(sum(Fraction(blk[i]) * h[i][k] for i in range(g)) * inv_sqrt_g)
        return out

    def f32(fr: Fraction) -> Fraction:
        return Fraction(float(np.float32(float(fr))))

    def quant(rows, per_token):
        rot_rows = [rot(r) for r in rows]
        if per_token:
            scales = [f32(max(abs(v) for v in r) / 127) for r in rot_rows]
        else:
            s = f32(max(abs(v) for r in rot_rows for v in r) / 127)
            scales = [s] * len(rot_rows)
        codes = [[0 if s == 0 else max(-127, min(127, _round_half_even(v / s))) for v in r]
                 for r, s in zip(rot_rows, scales)]
        return codes, scales

    xc, sx = quant(x, True)
    wc, sw = quant(w, False)
    y = []
    for m in range(len(x)):
        row = []
        for n in range(len(w)):
            acc = sum(a * b for a, b in zip(xc[m], wc[n]))
            row.append(acc * sx[m] * sw[0] + Fraction(bias[n]))
        y.append(row)
    return y


@pytest.mark.parametrize("g", [4, 16])
def test_linear_matches_exact_rational_pipeline(g):
    rng = np.random.default_rng(21 + g)
    K = 2 * g
    x = rng.standard_normal((3, K)).astype(np.float32).astype(np.float64)
    x[1, 3] *= 40.0  # an outlier channel
    w = (rng.standard_normal((4, K)) * 0.02).astype(np.float32).astype(np.float64)
    bias = (rng.standard_normal(4) * 0.01).astype(np.float32).astype(np.float64)
    exact = _exact_linear(x.tolist(), w.tolist(), bias.tolist(), g)
    wq, s_w = oracle.prepare_weight(w, g)
    y = oracle.linear(x, wq, s_w, g, bias)
    for m in range(3):
        for n in range(4):
            e = float(exact[m][n])
            assert abs(y[m, n] - e) <= 1e-14 * max(1.0, abs(e))


def test_zero_input_gives_zero_then_bias():
    d, _, w = _tiny()
    wq, s_w = oracle.prepare_weight(w, 256)
    x = np.zeros((4, 256))
    y = oracle.linear(x, wq, s_w, 256)
    assert np.all(y == 0.0)
    bias = oracle.bf16_to_f64(synth.f32_to_bf16_bits(np.linspace(-1, 1, 256).astype(np.float32)))
    yb = oracle.linear(x, wq, s_w, 256, bias)
    assert np.array_equal(yb, np.broadcast_to(bias, yb.shape))


def test_oracle_is_deterministic():
    d, x, w = _tiny()
    wq, s_w = oracle.prepare_weight(w, 256)
    y1 = oracle.linear(x, wq, s_w, 256)
    y2 = oracle.linear(x, wq, s_w, 256)
    assert np.array_equal(y1, y2)


def test_rotation_lowers_error_on_outlier_tokens():
    # the pages' reason for the rotation: without it one outlier channel sets
    # the scale of the whole token (InvokeAI "int8 Compute", "What stays on the
    # default path"). Same pipeline with g = 1 (R = I) as the control.
    d, x, w = _tiny()
    exact = x @ w.T
    wq, s_w = oracle.prepare_weight(w, 256)
    err_rot = oracle.nrmse(oracle.linear(x, wq, s_w, 256), exact)
    wq1, s_w1 = oracle.prepare_weight(w, 1)
    err_plain = oracle.nrmse(oracle.linear(x, wq1, s_w1, 1), exact)
    assert err_rot < 0.5 * err_plain
    assert err_rot < 2e-2


def test_to_bf16_rne_ties():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties to even (1.0)
    vals = np.array([1.0, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -2.5])
    bits = oracle.to_bf16_rne(vals)
    back = synth.bf16_bits_to_f32(bits).astype(np.float64).tolist()
    assert back == [1.0, 1.0, 1.0 + 2 * 2.0**-7, -2.5]


def test_nrmse_definition():
    ref = np.array([3.0, 4.0])
    assert oracle.nrmse(ref, ref) == 0.0
    assert oracle.nrmse(np.array([3.0, 4.0 + 0.5]), ref) == pytest.approx(0.1)


# ---------------------------------------------------------------- variants
# FP16 compute dtype, per-output-channel weight scale, exact-erf GELU.


def _bf16_from_definition(bits: int) -> float:
    """bfloat16 decoded by hand: sign, 8-bit exponent (bias 127), 7-bit fraction (the upper
    half of an IEEE binary32 word)."""
    s = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 7) & 0xFF
    f = bits & 0x7F
    if e == 0:
        return s * f * 2.0**-133
    if e == 255:
        return s * float("inf") if f == 0 else float("nan")
    return s * (1.0 + f / 128.0) * 2.0 ** (e - 127)


@pytest.mark.parametrize("bits,value", [(0x3F80, 1.0), (0xC000, -2.0), (0x3FFF, 1.9921875),
                                        (0x7F7F, (2.0 - 2.0**-7) * 2.0**127), (0x0001, 2.0**-133),
                                        (0x007F, 127 * 2.0**-133), (0x0080, 2.0**-126), (0x4049, 3.140625),
                                        (0xBE4D, -0.2001953125), (0x8000, -0.0), (0x7F80, float("inf"))])
def test_bf16_widening_follows_the_format(bits, value):
    got = float(oracle.bf16_to_f64(np.array([bits], np.uint16))[0])
    assert got == value == _bf16_from_definition(bits)
    assert np.signbit(got) == bool(bits & 0x8000)


def test_bf16_widening_of_every_finite_pattern():
    bits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    got = oracle.bf16_to_f64(bits[finite])
    want = np.array([_bf16_from_definition(int(b)) for b in bits[finite]])
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), (bits[finite] & 0x8000) != 0)


def _f16_from_definition(bits: int) -> float:
    """IEEE binary16 decoded by hand: sign, 5-bit exponent (bias 15), 10-bit fraction."""
    s = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 10) & 0x1F
    f = bits & 0x3FF
    if e == 0:
        return s * f * 2.0**-24
    if e == 31:
        return s * float("inf") if f == 0 else float("nan")
    return s * (1.0 + f / 1024.0) * 2.0 ** (e - 15)


@pytest.mark.parametrize("bits", [0x3C00, 0xC000, 0x7BFF, 0x0001, 0x03FF, 0x0400, 0x3555, 0x8000, 0x5640, 0xB4CD])
def test_f16_widening_follows_the_format(bits):
    got = float(oracle.f16_to_f64(np.array([bits], np.uint16))[0])
    assert got == _f16_from_definition(bits)
    assert np.signbit(got) == bool(bits & 0x8000)


def test_to_f16_rne_ties_and_range():
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: ties go to the even fraction (1.0)
    cases = {1.0 + 2.0**-11: 0x3C00, 1.0 + 3 * 2.0**-11: 0x3C02, -2.5: 0xC100, 65504.0: 0x7BFF,
             2.0**-24: 0x0001, 2.0**-25: 0x0000, 3 * 2.0**-25: 0x0002, 65520.0: 0x7C00}
    got = oracle.to_f16_rne(np.array(list(cases), np.float64))
    assert [int(b) for b in got] == list(cases.values())


def test_gelu_closed_forms():
    # Phi(1), Phi(2) of the standard normal CDF (tabulated constants)
    phi1 = 0.8413447460685429
    phi2 = 0.9772498680518208
    y = oracle.gelu_erf(np.array([0.0, 1.0, -1.0, 2.0, -2.0, 12.0, -12.0]))
    assert y[0] == 0.0
    assert abs(y[1] - phi1) < 1e-15 and abs(y[2] - (-(1.0 - phi1))) < 1e-15
    assert abs(y[3] - 2 * phi2) < 1e-15 and abs(y[4] - (-2 * (1.0 - phi2))) < 1e-15
    assert y[5] == 12.0 and abs(y[6]) < 1e-30


def test_gelu_odd_part_is_identity():
    # y Phi(y) - (-y) Phi(-y) = y (Phi(y) + Phi(-y)) = y, for every y
    x = np.random.default_rng(3).standard_normal(1000) * 4
    np.testing.assert_allclose(oracle.gelu_erf(x) - oracle.gelu_erf(-x), x, rtol=0, atol=1e-14)


def test_per_channel_weight_scale_follows_rows():
    # rows that are power-of-two multiples of one row: identical codes, scales
    # in the same ratios (a scale taken along the wrong axis breaks both)
    rng = np.random.default_rng(4)
    base = rng.standard_normal(256)
    w = np.stack([base * 2.0**k for k in range(-3, 5)])
    wq, sw = oracle.prepare_weight_per_channel(w, 256)
    assert sw.dtype == np.float32 and sw.shape == (8,)
    for n in range(1, 8):
        assert np.array_equal(wq[n], wq[0])
        assert sw[n] == np.float32(sw[0] * 2.0**n)
    assert np.all(np.max(np.abs(wq.astype(np.int32)), axis=1) == 127)
    # and the scale of a row is max |row of W R| / 127
    wr = oracle.rotate(w, 256)
    np.testing.assert_array_equal(sw, (np.max(np.abs(wr), axis=1) / 127).astype(np.float32))


def test_dequant_per_channel_hand_case_and_tensorwise_limit():
    acc = np.array([[1, 2], [3, 4]], np.int32)
    y = oracle.dequant_per_channel(acc, np.array([1.0, 0.5]), np.array([2.0, 4.0]), np.array([0.5, -1.0]))
    np.testing.assert_array_equal(y, [[2.5, 7.0], [3.5, 7.0]])
    rng = np.random.default_rng(5)
    acc = rng.integers(-1000, 1000, (5, 7)).astype(np.int32)
    sx = rng.random(5).astype(np.float32)
    np.testing.assert_array_equal(oracle.dequant_per_channel(acc, sx, np.full(7, 0.25, np.float32)),
                                  oracle.dequant(acc, sx, np.float32(0.25)))


def test_linear_ex_reduces_to_its_parts():
    # the composed variant equals its definition step by step, and with no
    # options it is exactly the plain layer
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 256))
    w = rng.standard_normal((8, 256)) * 0.02
    b = rng.standard_normal(8) * 0.01
    z = rng.standard_normal((5, 8)) * 0.05
    wq, sw = oracle.prepare_weight(w, 256)
    np.testing.assert_array_equal(oracle.linear_ex(x, wq, sw, 256, b), oracle.linear(x, wq, sw, 256, b))
    y0 = oracle.linear(x, wq, sw, 256, b)
    np.testing.assert_array_equal(oracle.linear_ex(x, wq, sw, 256, b, addend=z), y0 + z)
    np.testing.assert_array_equal(oracle.linear_ex(x, wq, sw, 256, b, addend=z, gelu=True), oracle.gelu_erf(y0 + z))
    wqc, swc = oracle.prepare_weight_per_channel(w, 256)
    xq, sx = oracle.quant_act(x, 256)
    ref = oracle.gemm_s32(xq, wqc) * (sx[:, None].astype(np.float64) * swc[None, :].astype(np.float64)) + b
    np.testing.assert_array_equal(oracle.linear_ex(x, wqc, swc, 256, b), ref)


def test_addend_hand_case():
    # one token, one output: x = 4 e_0 in a 256-group -> codes 127 * sign pattern / 127 ...
    # built so the accumulator is known: x rotated is c/16 * H[0,:] = all +c/16, so s_x = c/(16*127)
    # and every code is 127; a weight row equal to e_0 rotates to all +1/16, codes 127, s_w = 1/(16*127)
    x = np.zeros((1, 256))
    x[0, 0] = 4.0
    w = np.zeros((1, 256))
    w[0, 0] = 1.0
    wq, sw = oracle.prepare_weight(w, 256)
    y = oracle.linear_ex(x, wq, sw, 256, bias=np.array([0.5]), addend=np.array([[-0.25]]))
    # acc = 256 * 127^2; y = acc * s_x * s_w + 0.5 - 0.25 = x . w + 0.25 = 4.25 (to float32 rounding of the scales)
    assert abs(y[0, 0] - 4.25) < 1e-6
