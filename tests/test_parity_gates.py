"""The parity gates reject what they must: negative controls on the CPU.

The GPU tests compare the CUDA path with the oracle through the helpers in
tests/parity.py. Here those helpers are fed planted failures -- an all-zero
output (rejected at 100% error), a non-finite value, codes off by more than
one or away from a rounding tie, a scale off by more than the tolerance -- and
must refuse every one, so that a passing GPU test cannot come from a gate that
accepts anything.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from parity import NRMSE_TOL, check_codes, check_output_elementwise, nrmse


def _case(seed=0, M=16, K=256, g=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    xr = oracle.rotate(x, g)
    q, s = oracle.quantize_per_token(xr)
    return xr, q, s


def test_zero_output_is_rejected_at_full_error():
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((32, 64))
    assert nrmse(np.zeros_like(ref), ref) == pytest.approx(1.0)
    assert not nrmse(np.zeros_like(ref), ref) <= NRMSE_TOL


def test_non_finite_output_is_rejected():
    rng = np.random.default_rng(2)
    ref = rng.standard_normal((8, 8))
    y = ref.copy()
    y[3, 4] = np.nan
    assert not nrmse(y, ref) <= NRMSE_TOL
    y[3, 4] = np.inf
    assert not nrmse(y, ref) <= NRMSE_TOL


def test_small_rounding_noise_passes():
    # bf16 output rounding alone stays well inside the bound
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((64, 64))
    y = oracle.bf16_to_f64(oracle.to_bf16_rne(ref))
    assert nrmse(y, ref) <= NRMSE_TOL


def test_identical_codes_pass():
    xr, q, s = _case()
    check_codes(q.copy(), s.copy(), xr, q, s)


def test_code_off_by_two_is_rejected():
    xr, q, s = _case()
    bad = q.copy()
    bad[2, 5] = np.clip(int(bad[2, 5]) + 2, -127, 127) if bad[2, 5] < 120 else bad[2, 5] - 2
    with pytest.raises(AssertionError):
        check_codes(bad, s, xr, q, s)


def test_code_off_by_one_away_from_a_tie_is_rejected():
    # large enough that one differing code is under the 1e-4 mismatch fraction:
    # only the near-tie condition can reject it
    xr, q, s = _case(M=64, K=2048)
    quot = xr / s[:, None].astype(np.float64)
    frac = np.abs(np.abs(quot - np.floor(quot)) - 0.5)
    m, k = np.unravel_index(np.argmax(frac), frac.shape)  # the element farthest from a tie
    bad = q.copy()
    bad[m, k] = bad[m, k] + (1 if bad[m, k] < 127 else -1)
    with pytest.raises(AssertionError, match="near-tie"):
        check_codes(bad, s, xr, q, s)


def test_scale_off_by_more_than_the_tolerance_is_rejected():
    xr, q, s = _case()
    bad = s.copy()
    bad[7] = np.float32(bad[7] * (1 + 1e-5))
    with pytest.raises(AssertionError):
        check_codes(q, bad, xr, q, s)


def test_code_outside_the_symmetric_range_is_rejected():
    xr, q, s = _case(M=64, K=2048)
    bad = q.astype(np.int16)
    i = np.argmax(q.astype(np.int32))
    assert q.flat[i] == 127
    bad.flat[i] = 128  # one step off, under the mismatch fraction: only the range check can reject it
    with pytest.raises(AssertionError, match="range|tie"):
        check_codes(bad, s, xr, q, s)


def _simulated_epilogue(seed=5, M=48, N=40, K=3072, gelu=False, out="bf16", addend=False):
    """A float32 epilogue as the kernel computes it (float(acc) * (s_x * s_w) + bias, then the
    output rounding), on random codes' accumulators; returns the inputs and the output."""
    from scipy.special import erf

    rng = np.random.default_rng(seed)
    acc = rng.integers(-127 * 127 * 8, 127 * 127 * 8, size=(M, N)).astype(np.int64)
    acc[0, :4] = [0, K * 127 * 127, -K * 127 * 127, 1]
    sx = (rng.random(M) * 0.05 + 1e-3).astype(np.float32)
    sx[1] = 0.0
    sw = np.float32(2.3e-4)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float32)
    add = (rng.standard_normal((M, N)) * 0.05).astype(np.float32) if addend else None
    z = acc.astype(np.float32) * (sx[:, None] * sw) + bias[None, :]
    if add is not None:
        z = z + add
    if gelu:
        z = (np.float32(0.5) * z * (np.float32(1.0) + erf(z / np.float32(np.sqrt(2.0))).astype(np.float32)))
    z64 = z.astype(np.float64)
    y = oracle.bf16_to_f64(oracle.to_bf16_rne(z64)) if out == "bf16" else oracle.f16_to_f64(oracle.to_f16_rne(z64))
    return acc, sx, sw, bias, add, y


@pytest.mark.parametrize("gelu,out,addend", [(False, "bf16", False), (True, "bf16", True), (False, "f16", True),
                                             (True, "f16", False)])
def test_elementwise_gate_passes_a_float32_epilogue(gelu, out, addend):
    acc, sx, sw, bias, add, y = _simulated_epilogue(gelu=gelu, out=out, addend=addend)
    assert check_output_elementwise(y, acc, sx, sw, bias, add, gelu=gelu, out=out) <= 1.0


@pytest.mark.parametrize("factor", [1.02, 0.0, -1.0])
def test_elementwise_gate_rejects_one_wrong_element(factor):
    acc, sx, sw, bias, add, y = _simulated_epilogue()
    bad = y.copy()
    i, j = 17, 23
    assert abs(bad[i, j]) > 1e-3
    bad[i, j] *= factor
    with pytest.raises(AssertionError, match=r"output element \(17, 23\)"):
        check_output_elementwise(bad, acc, sx, sw, bias)
    # the same corruption passes the NRMSE gate: it is the element-wise bound that catches it
    ref = acc * (sx.astype(np.float64)[:, None] * np.float64(sw)) + bias.astype(np.float64)[None, :]
    assert nrmse(bad, ref) <= NRMSE_TOL or factor != 1.02


def test_elementwise_gate_rejects_a_dropped_bias_and_a_wrong_scale():
    acc, sx, sw, bias, add, y = _simulated_epilogue()
    with pytest.raises(AssertionError):
        check_output_elementwise(y, acc, sx, sw, None)
    with pytest.raises(AssertionError):
        check_output_elementwise(y, acc, sx, np.float32(sw * 1.001), bias)
