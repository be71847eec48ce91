"""Pins of the INT8 attention oracle against facts fixed by the mathematics.

Each test checks the oracle against something independent of its own code: a
library softmax and attention routine, closed forms (one key, identical keys,
a constant value vector), a brute-force evaluation in plain Python on a tiny
case, and the rounding bound of the int8 logits around the exact ones (which
also pins the rotation: it must leave Q K^T unchanged).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import scipy.special

import oracle


def _qkv(seed=0, bh=2, sq=7, skv=9, d=128, qk=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((bh, sq, d)) * qk
    k = rng.standard_normal((bh, skv, d))
    v = rng.standard_normal((bh, skv, d))
    return q, k, v


def test_softmax_matches_scipy_and_sums_to_one():
    rng = np.random.default_rng(1)
    s = rng.standard_normal((3, 5, 40)) * 10
    p = oracle.softmax(s)
    np.testing.assert_allclose(p, scipy.special.softmax(s, axis=-1), rtol=1e-13, atol=0)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(p >= 0)


def test_exact_attention_matches_torch_sdpa():
    import torch

    q, k, v = _qkv(2, sq=5, skv=11, d=64)
    o = oracle.attention_exact(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                                           torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_single_key_returns_its_value():
    q, k, v = _qkv(3, sq=4, skv=1)
    o = oracle.attention_int8(q, k, v)
    assert np.array_equal(o, np.broadcast_to(v, o.shape))


def test_identical_keys_average_the_values():
    q, k, v = _qkv(4, sq=3, skv=6)
    k[:] = k[:, :1, :]  # every key the same: uniform weights
    o = oracle.attention_int8(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape), rtol=0, atol=1e-14)


def test_constant_value_vector_is_returned():
    q, k, v = _qkv(5, sq=5, skv=8)
    v[:] = v[:, :1, :]
    o = oracle.attention_int8(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v[:, :1, :], o.shape), rtol=0, atol=1e-14)


def test_zero_output_control_is_rejected_at_full_error():
    q, k, v = _qkv(6)
    o = oracle.attention_int8(q, k, v)
    assert oracle.nrmse(np.zeros_like(o), o) == pytest.approx(1.0)


def _brute_force(q, k, v, scale):
    """Tiny case in plain Python: D = 4, rotation by the 4x4 Hadamard matrix written out."""
    h = [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]

    def quant(row):
        r = [sum(row[c] * h[c][j] for c in range(4)) / 2.0 for j in range(4)]  # row . H / sqrt(4)
        amax = max(abs(x) for x in r)
        s = float(np.float32(amax / 127.0))
        codes = [0 if s == 0 else max(-127, min(127, round(x / s))) for x in r]  # round(): ties to even
        return codes, s

    out = []
    for qi in q:
        cq, sq = quant(qi)
        logits = []
        for kj in k:
            ck, sk = quant(kj)
            logits.append(sum(a * b for a, b in zip(cq, ck)) * sq * sk * scale)
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        tot = sum(e)
        out.append([sum(e[j] * v[j][c] for j in range(len(k))) / tot for c in range(4)])
    return np.array(out)


def test_brute_force_tiny_case():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((3, 4)) * 3
    k = rng.standard_normal((5, 4)) * 2
    v = rng.standard_normal((5, 4))
    k[2] = 0.0  # an all-zero key: scale 0, codes 0, logit 0
    o = oracle.attention_int8(q, k, v, softmax_scale=0.5, g=4)
    np.testing.assert_allclose(o, _brute_force(q.tolist(), k.tolist(), v.tolist(), 0.5), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("qk", [1.0, 4.0])
def test_int8_logits_within_the_rounding_bound_of_the_exact_ones(qk):
    # codes differ from the rotated values by at most half a step, so
    # |S_int8 - S| <= scale * sum_r (|q'_r| s_k / 2 + |k'_r| s_q / 2 + s_q s_k / 4),
    # with S = q . k * scale (the rotation leaves the dot product unchanged)
    q, k, v = _qkv(8, sq=16, skv=24, qk=qk)
    q[0, 3, 17] *= 40.0  # an outlier channel in one token
    scale = 1.0 / math.sqrt(128)
    _, parts = oracle.attention_int8(q, k, v, return_parts=True)
    qr, kr = oracle.rotate(q, 128), oracle.rotate(k, 128)
    exact = (q @ np.swapaxes(k, -1, -2)) * scale
    sq = parts["sq"].astype(np.float64)[..., :, None]
    sk = parts["sk"].astype(np.float64)[..., None, :]
    bound = scale * (np.abs(qr).sum(-1)[..., :, None] * sk / 2 + np.abs(kr).sum(-1)[..., None, :] * sq / 2
                     + 128 * sq * sk / 4)
    err = np.abs(parts["s"] - exact)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-12)
    # and the bound is not vacuous: the int8 logits are far closer than the logits' spread
    assert err.max() < 0.05 * np.abs(exact).max()


def test_codes_and_scales_are_the_linear_layer_rule():
    q, k, v = _qkv(9, sq=6, skv=6)
    _, parts = oracle.attention_int8(q, k, v, return_parts=True)
    qc, sq = oracle.quant_act(q.reshape(-1, 128), 128)
    assert np.array_equal(parts["qc"].reshape(-1, 128), qc) and np.array_equal(parts["sq"].reshape(-1), sq)
    assert np.all(np.abs(parts["qc"]).max(axis=-1) == 127)


def test_attention_is_close_to_exact_attention():
    # sanity, not parity: int8 logits move the output little at unit logit scale
    q, k, v = _qkv(10, bh=4, sq=64, skv=256)
    err = oracle.nrmse(oracle.attention_int8(q, k, v), oracle.attention_exact(q, k, v))
    assert err < 0.02
