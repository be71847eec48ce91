"""Parity of the INT8 attention kernels (through the C ABI) with the CPU oracle, on a B200.

The query and key codes and scales the call leaves in its workspace are
checked against the oracle's (near-ties only), then every output element
against the oracle's softmax(S) V evaluated on the kernel's own codes and
scales, within the rounding bound of the kernel's arithmetic:

    |O - O_ref| <= 2^-8 |O_ref|                       (output rounded to bf16)
                 + (2^-8 + eps_t) * sum_k P_ref[k] |V_k|   (P rounded to bf16;
                                                       float32 logits and exp2)
bf16 keeps 8 significant bits, so one round-to-nearest-even moves a value by
at most 2^-8 of itself (half an ulp at the bottom of a binade); the P V
numerator carries that on each p_k, while the row sum uses the unrounded p_k.
with eps_t = 1e-5 * (1 + max |S_ref| log2 e). The NRMSE against the oracle's
own result is also bounded (3e-3).
"""

from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from parity import check_codes

pytestmark = pytest.mark.gpu

ATTN_NRMSE_TOL = 3e-3


@pytest.fixture(scope="module")
def cr():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_rotated_int8_token_b200 as cr

    cr.lib()
    return cr


def _bf16(x):
    import synth

    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


def _to_dev(bits):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _from_dev(t):
    import torch

    u16 = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ws_layout(BH, Sq, Skv):
    up = lambda v, a: (v + a - 1) // a * a  # noqa: E731
    qq = 256
    sq = up(qq + BH * Sq * 128, 256)
    kq = up(sq + 4 * BH * Sq, 1024)
    sk = up(kq + BH * Skv * 128, 256)
    return qq, sq, kq, sk


def _run(cr, q, k, v, scale=None, rows=None):
    """q [BH, Sq, 128], k/v [BH, Skv, 128] float32 values (rounded to bf16 here). Returns
    the kernel's O (float64) and its codes/scales from the workspace, and the bf16 inputs."""
    import torch

    BH, Sq, _ = q.shape
    Skv = k.shape[1]
    qb, kb, vb = _bf16(q), _bf16(k), _bf16(v)
    ws = torch.empty(cr.convrot_attention_workspace_bytes(BH, Sq, Skv), dtype=torch.uint8, device="cuda")
    O = cr.convrot_attention_int8(_to_dev(qb), _to_dev(kb), _to_dev(vb), softmax_scale=scale, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    wsn = ws.cpu().numpy()
    o_qq, o_sq, o_kq, o_sk = _ws_layout(BH, Sq, Skv)
    qc = wsn[o_qq:o_qq + BH * Sq * 128].view(np.int8).reshape(BH, Sq, 128)
    sq = wsn[o_sq:o_sq + 4 * BH * Sq].view(np.float32).reshape(BH, Sq)
    kc = wsn[o_kq:o_kq + BH * Skv * 128].view(np.int8).reshape(BH, Skv, 128)
    sk = wsn[o_sk:o_sk + 4 * BH * Skv].view(np.float32).reshape(BH, Skv)
    return _from_dev(O), qc, sq, kc, sk, (qb, kb, vb)


def _check(cr, q, k, v, scale=None, heads=None, rows=None):
    BH, Sq, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o, qc, sq, kc, sk, (qb, kb, vb) = _run(cr, q, k, v, scale)
    heads = range(BH) if heads is None else heads
    for h in heads:
        r = np.arange(Sq) if rows is None else rows
        qf = oracle.bf16_to_f64(qb[h][r])
        kf = oracle.bf16_to_f64(kb[h])
        vf = oracle.bf16_to_f64(vb[h])
        # codes and scales against the oracle's (near-ties only)
        qr, kr = oracle.rotate(qf, 128), oracle.rotate(kf, 128)
        cq_ref, sq_ref = oracle.quantize_per_token(qr)
        ck_ref, sk_ref = oracle.quantize_per_token(kr)
        check_codes(qc[h][r], sq[h][r], qr, cq_ref, sq_ref)
        check_codes(kc[h], sk[h], kr, ck_ref, sk_ref)
        # every output element against softmax(S) V on the kernel's own codes and scales
        s_ref = oracle.attention_logits(qc[h][r], sq[h][r], kc[h], sk[h], scale)
        p_ref = oracle.softmax(s_ref)
        o_ref = p_ref @ vf
        pv = p_ref @ np.abs(vf)
        eps_t = 1e-5 * (1.0 + np.abs(s_ref).max() * math.log2(math.e))
        bound = 2.0**-8 * np.abs(o_ref) + (2.0**-8 + eps_t) * pv + 1e-7
        y = o[h][r]
        assert np.all(np.isfinite(y))
        ratio = np.abs(y - o_ref) / bound
        assert ratio.max() <= 1.0, f"head {h}: element {np.unravel_index(np.argmax(ratio), ratio.shape)} " \
                                   f"off by {ratio.max():.2f} x its bound"
        # and the oracle's own result (its own codes)
        o_own = oracle.attention_int8(qf, kf, vf, softmax_scale=scale)
        err = oracle.nrmse(y, o_own)
        assert err <= ATTN_NRMSE_TOL, f"head {h}: NRMSE {err}"
    return o


def _qkv(seed, BH, Sq, Skv, qk=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((BH, Sq, 128)).astype(np.float32) * qk
    k = rng.standard_normal((BH, Skv, 128)).astype(np.float32)
    v = rng.standard_normal((BH, Skv, 128)).astype(np.float32)
    return q, k, v


@pytest.mark.parametrize("BH,Sq,Skv", [(2, 256, 256), (1, 128, 128), (3, 200, 300), (2, 1, 1), (1, 5, 129),
                                       (2, 130, 1000)])
def test_attention_matches_oracle_ragged(cr, BH, Sq, Skv):
    q, k, v = _qkv(BH * 1000 + Sq + Skv, BH, Sq, Skv)
    _check(cr, q, k, v)


def test_attention_rescales_when_later_keys_raise_the_maximum(cr):
    # logits that grow block by block: the running maximum moves up several times
    # by more than the rescale threshold
    q, k, v = _qkv(11, 2, 256, 640, qk=4.0)
    k *= np.linspace(0.2, 3.0, 640, dtype=np.float32)[None, :, None]
    _check(cr, q, k, v)


def test_attention_large_logits_and_outliers(cr):
    # the pages' error case: a logit scale of 4, plus an outlier channel in Q
    q, k, v = _qkv(12, 2, 384, 384, qk=4.0)
    q[:, :, 7] *= 30.0
    _check(cr, q, k, v)


def test_attention_zero_query_rows_average_the_values(cr):
    q, k, v = _qkv(13, 1, 128, 200)
    q[0, 3] = 0.0  # scale 0, codes 0: uniform weights over the keys
    o = _check(cr, q, k, v)
    vb = oracle.bf16_to_f64(_bf16(v[0]))
    np.testing.assert_allclose(o[0, 3], vb.mean(axis=0), rtol=0, atol=2e-2)


def test_attention_full_shape_sampled_rows(cr):
    # 4096 image + 128 prefix tokens, 32 heads, head dim 128; sampled query rows of a few heads
    q, k, v = _qkv(14, 32, 4224, 4224)
    rows = np.unique(np.concatenate([np.arange(64), np.random.default_rng(0).choice(4224, 96, replace=False),
                                     np.arange(4224 - 64, 4224)]))
    _check(cr, q, k, v, heads=[0, 13, 31], rows=rows)


def test_attention_deterministic(cr):
    import torch

    q, k, v = _qkv(15, 2, 256, 384)
    Q, K, V = (_to_dev(_bf16(t)) for t in (q, k, v))
    o1 = cr.convrot_attention_int8(Q, K, V)
    o2 = cr.convrot_attention_int8(Q, K, V)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_attention_rejects_bad_arguments(cr):
    import torch

    L = cr.lib()
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    x = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    # D must be 128
    assert L.convrot_attention_int8(x.data_ptr(), x.data_ptr(), x.data_ptr(), 1, 8, 8, 64, 0.125, x.data_ptr(),
                                    ws.data_ptr(), ws.numel(), None) == 2
    y = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    # no keys; a non-positive scale
    assert L.convrot_attention_int8(y.data_ptr(), y.data_ptr(), y.data_ptr(), 1, 8, 0, 128, 0.1, y.data_ptr(),
                                    ws.data_ptr(), ws.numel(), None) == 1
    assert L.convrot_attention_int8(y.data_ptr(), y.data_ptr(), y.data_ptr(), 1, 8, 8, 128, 0.0, y.data_ptr(),
                                    ws.data_ptr(), ws.numel(), None) == 1
    # workspace too small
    assert L.convrot_attention_int8(y.data_ptr(), y.data_ptr(), y.data_ptr(), 1, 8, 8, 128, 0.1, y.data_ptr(),
                                    ws.data_ptr(), 256, None) == 3
