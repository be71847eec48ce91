"""Parity of the layer's variants with the CPU oracle, on a B200, through the C ABI.

Variants (convrot_*_ex): the FP16 compute dtype (X, W, bias and Y in fp16),
one weight scale per output channel, the exact-erf GELU fused into the
epilogue, an addend computed beside the int8 layer (a LoRA's output), and
strided rows of X, Y and the addend. Each case runs in the same launch configuration as the default
layer (CTA-pair GEMM for M > 64, the weight-streaming GEMM for M <= 64) and is
compared with the oracle's float64 result on sampled token rows.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from parity import NRMSE_TOL, check_codes, check_output_elementwise, nrmse
from test_abi import linear_ws_layout

pytestmark = pytest.mark.gpu

BF16, F16 = 0, 1
TENSOR, CHANNEL = 0, 1
NONE, GELU = 0, 1


@pytest.fixture(scope="module")
def cr():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_rotated_int8_token_b200 as cr

    cr.lib()
    return cr


def _rows_sample(M: int, n: int = 384, seed: int = 1) -> np.ndarray:
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(128, M - 128), n - 256, replace=False)
    return np.unique(np.concatenate([np.arange(128), mid, np.arange(M - 128, M)]))


def _as_dtype_bits(bf16_bits: np.ndarray, dtype: int) -> np.ndarray:
    """The workload's values in the compute dtype: bf16 bits as they are, or the
    same values rounded to fp16 (bits)."""
    if dtype == BF16:
        return np.asarray(bf16_bits, np.uint16)
    return synth.bf16_bits_to_f32(bf16_bits).astype(np.float16).view(np.uint16)


def _to_f64(bits: np.ndarray, dtype: int) -> np.ndarray:
    return oracle.bf16_to_f64(bits) if dtype == BF16 else oracle.f16_to_f64(bits)


def _to_torch(bits: np.ndarray, dtype: int):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if dtype == BF16 else torch.float16)


def _from_torch(t, dtype: int) -> np.ndarray:
    import torch

    u16 = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return _to_f64(u16, dtype)


def _kernel_codes(ws, M: int, K: int, rows: np.ndarray):
    """The token scales and activation codes a layer call left in its workspace (sampled rows)."""
    wsn = ws.cpu().numpy()
    lay = linear_ws_layout(M, K)
    sx = wsn[lay["scale"]:lay["scale"] + 4 * M].view(np.float32)[rows]
    xq = wsn[lay["codes"]:lay["codes"] + M * K].view(np.int8).reshape(M, K)[rows]
    return xq, sx


def _check_elementwise(ws, M, K, rows, x_rows64, w64, g, mode, Wq, sw, y, bias64, addend64, act, dtype):
    """The call's codes and scales against the oracle's (near-ties only), then every output
    element against the oracle's arithmetic on the kernel's own codes and scales."""
    xq_gpu, sx_gpu = _kernel_codes(ws, M, K, rows)
    xr = oracle.rotate(x_rows64, g)
    q_ref, s_ref = oracle.quantize_per_token(xr)
    check_codes(xq_gpu, sx_gpu, xr, q_ref, s_ref)
    wq_gpu = Wq.cpu().numpy()
    sw_gpu = sw.cpu().numpy().reshape(-1)
    wr = oracle.rotate(w64, g)
    if mode == CHANNEL:
        wq_ref, sw_ref = oracle.quantize_per_token(wr)
        check_codes(wq_gpu, sw_gpu, wr, wq_ref, sw_ref)
        sw_use = sw_gpu
    else:
        wq_ref, sw_ref = oracle.quantize_tensorwise(wr)
        check_codes(wq_gpu, sw_gpu, wr, wq_ref, np.array([sw_ref]), per_token=False)
        sw_use = float(sw_gpu[0])
    return check_output_elementwise(y, oracle.gemm_s32(xq_gpu, wq_gpu), sx_gpu, sw_use, bias64, addend64,
                                    gelu=(act == GELU), out="bf16" if dtype == BF16 else "f16")


def _oracle_layer(x, w, g, mode, bias, act):
    if mode == CHANNEL:
        wq, sw = oracle.prepare_weight_per_channel(w, g)
    else:
        wq, sw = oracle.prepare_weight(w, g)
    xq, sx = oracle.quant_act(x, g)
    acc = oracle.gemm_s32(xq, wq)
    y = oracle.dequant_per_channel(acc, sx, sw, bias) if mode == CHANNEL else oracle.dequant(acc, sx, sw, bias)
    return oracle.gelu_erf(y) if act == GELU else y


CASES = [
    ("tiny", BF16, CHANNEL, NONE),
    ("tiny", F16, TENSOR, NONE),
    ("tiny", BF16, TENSOR, GELU),
    ("tiny", F16, CHANNEL, GELU),
    ("dit_qkv_1024", F16, TENSOR, NONE),
    ("dit_qkv_1024", BF16, CHANNEL, NONE),
    ("dit_mlp_up_1024", BF16, TENSOR, GELU),
    ("dit_mlp_up_1024", F16, CHANNEL, GELU),
    ("textenc_m16", BF16, CHANNEL, GELU),
    ("textenc_m1", BF16, CHANNEL, NONE),
    ("textenc_m16", F16, TENSOR, NONE),
    ("textenc_m128", F16, CHANNEL, NONE),
]


@pytest.mark.parametrize("name,dtype,mode,act", CASES)
def test_linear_ex_matches_oracle(cr, name, dtype, mode, act):
    import torch

    d = synth.make_workload(name)
    g = d["workload"].g
    xb = _as_dtype_bits(d["x"], dtype)
    wb = _as_dtype_bits(d["w"], dtype)
    bb = None if d["bias"] is None else _as_dtype_bits(d["bias"], dtype)
    Wq, sw = cr.convrot_prepare_weight_ex(_to_torch(wb, dtype), g, mode)
    X = _to_torch(xb, dtype)
    bias = None if bb is None else _to_torch(bb, dtype)
    M, K = xb.shape
    N = wb.shape[0]
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    Y = cr.convrot_linear_ex(X, Wq, sw, g, bias, act, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    assert Y.dtype == X.dtype and tuple(Y.shape) == (M, N)
    rows = _rows_sample(M)
    ref = _oracle_layer(_to_f64(xb[rows], dtype), _to_f64(wb, dtype), g, mode,
                        None if bb is None else _to_f64(bb, dtype), act)
    y = _from_torch(Y, dtype)[rows]
    assert np.all(np.isfinite(y))
    err = nrmse(y, ref)
    assert err <= NRMSE_TOL, f"{name} dtype={dtype} mode={mode} act={act}: NRMSE {err}"
    _check_elementwise(ws, M, K, rows, _to_f64(xb[rows], dtype), _to_f64(wb, dtype), g, mode, Wq, sw, y,
                       None if bb is None else _to_f64(bb, dtype), None, act, dtype)


@pytest.mark.parametrize("name,dtype", [("tiny", BF16), ("tiny", F16), ("dit_qkv_1024", BF16), ("textenc_m16", F16)])
def test_prepare_weight_per_channel_matches_oracle(cr, name, dtype):
    import torch

    d = synth.make_workload(name)
    g = d["workload"].g
    wb = _as_dtype_bits(d["w"], dtype)
    Wq, sw = cr.convrot_prepare_weight_ex(_to_torch(wb, dtype), g, CHANNEL)
    torch.cuda.synchronize()
    wr = oracle.rotate(_to_f64(wb, dtype), g)
    q_ref, s_ref = oracle.quantize_per_token(wr)
    check_codes(Wq.cpu().numpy(), sw.cpu().numpy(), wr, q_ref, s_ref)
    assert np.all(np.abs(Wq.cpu().numpy().astype(np.int32)).max(axis=1) == 127)


@pytest.mark.parametrize("name", ["tiny", "dit_qkv_1024", "textenc_m512"])
def test_quant_act_f16_matches_oracle(cr, name):
    import torch

    d = synth.make_workload(name)
    g = d["workload"].g
    xb = _as_dtype_bits(d["x"], F16)
    Xq, s = cr.convrot_quant_act_ex(_to_torch(xb, F16), g)
    torch.cuda.synchronize()
    xr = oracle.rotate(_to_f64(xb, F16), g)
    q_ref, s_ref = oracle.quantize_per_token(xr)
    check_codes(Xq.cpu().numpy(), s.cpu().numpy(), xr, q_ref, s_ref)


@pytest.mark.parametrize("name", ["dit_qkv_1024", "textenc_m16"])
def test_equal_channel_scales_reproduce_the_tensorwise_output(cr, name):
    # per-channel scales all equal to the tensor scale: the general epilogue
    # must give exactly the default epilogue's bits (same product, same rounding)
    import torch

    d = synth.make_workload(name)
    g = d["workload"].g
    W = _to_torch(d["w"], BF16)
    Wq, sw = cr.convrot_prepare_weight(W, g)
    X = _to_torch(d["x"], BF16)
    bias = None if d["bias"] is None else _to_torch(d["bias"], BF16)
    N = Wq.shape[0]
    Y0 = cr.convrot_linear(X, Wq, sw, g, bias)
    Y1 = cr.convrot_linear_ex(X, Wq, sw.repeat(N).contiguous(), g, bias, NONE)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))


def test_default_options_are_convrot_linear(cr):
    import torch

    d = synth.make_workload("tiny")
    g = d["workload"].g
    Wq, sw = cr.convrot_prepare_weight(_to_torch(d["w"], BF16), g)
    X = _to_torch(d["x"], BF16)
    Y0 = cr.convrot_linear(X, Wq, sw, g)
    Y1 = cr.convrot_linear_ex(X, Wq, sw, g, None, NONE)
    torch.cuda.synchronize()
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))


@pytest.mark.parametrize("name,M", [("pair", 192), ("smallm", 16)])
def test_gelu_epilogue_against_the_exact_function(cr, name, M):
    # zero input: every code and accumulator is 0, so each output is GELU(bias[n])
    # rounded once to fp16. The epilogue's erf (Abramowitz-Stegun 7.1.26) is
    # within 1.5e-7 of the exact one, so the output is within half an fp16 ulp
    # of the exact GELU plus 0.5 |y| 1.5e-7 (+ float32 rounding).
    import torch

    K, N, g = 256, 512, 256
    rng = np.random.default_rng(11)
    wb = (rng.standard_normal((N, K)) * 0.02).astype(np.float16).view(np.uint16)
    bvals = np.concatenate([np.linspace(-6.0, 6.0, N - 8), [0.0, -0.0, 1e-3, -1e-3, 30.0, -30.0, 2.5, -2.5]])
    bb = bvals.astype(np.float16).view(np.uint16)
    Wq, sw = cr.convrot_prepare_weight_ex(_to_torch(wb, F16), g, TENSOR)
    X = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    Y = cr.convrot_linear_ex(X, Wq, sw, g, _to_torch(bb, F16), GELU)
    torch.cuda.synchronize()
    y = _from_torch(Y, F16)
    ref = oracle.gelu_erf(oracle.f16_to_f64(bb))
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)  # fp16 ulp at |ref|
    bound = 0.5 * ulp + 0.5 * np.abs(oracle.f16_to_f64(bb)) * 2e-7 + 1e-7 * np.abs(ref)
    for m in (0, M // 2, M - 1):
        assert np.all(np.abs(y[m] - ref) <= bound + 1e-12), np.max(np.abs(y[m] - ref) - bound)


@pytest.mark.parametrize("name,dtype,act,x_pad", [("tiny", BF16, NONE, 64), ("dit_qkv_1024", F16, GELU, 64),
                                                  ("textenc_m16", BF16, GELU, 64), ("textenc_m128", F16, NONE, 64),
                                                  ("textenc_m16", BF16, GELU, 0), ("textenc_m1", BF16, GELU, 0)])
def test_strided_rows_and_addend_match_oracle(cr, name, dtype, act, x_pad):
    # X and Y live inside wider row-major buffers (row strides K + x_pad and
    # N + 40), the addend shares Y's stride; the oracle sees the dense values.
    # Dense bf16 rows of one token (x_pad 0, textenc_m1) take the one-kernel form.
    import torch

    d = synth.make_workload(name)
    g = d["workload"].g
    xb = _as_dtype_bits(d["x"], dtype)
    wb = _as_dtype_bits(d["w"], dtype)
    bb = None if d["bias"] is None else _as_dtype_bits(d["bias"], dtype)
    M, K = xb.shape
    N = wb.shape[0]
    rng = np.random.default_rng(21)
    zb = _as_dtype_bits(synth.f32_to_bf16_bits((rng.standard_normal((M, N)) * 0.05).astype(np.float32)), dtype)
    Wq, sw = cr.convrot_prepare_weight_ex(_to_torch(wb, dtype), g, TENSOR)
    ldx, ldy = K + x_pad, N + 40
    Xbig = _to_torch(np.zeros((M, ldx), np.uint16), dtype)
    Xbig[:, :K] = _to_torch(xb, dtype)
    Ybig = torch.full((M, ldy), float("nan"), dtype=Xbig.dtype, device="cuda")
    Zbig = torch.zeros((M, ldy), dtype=Xbig.dtype, device="cuda")
    Zbig[:, :N] = _to_torch(zb, dtype)
    X, Y, Z = Xbig[:, :K], Ybig[:, :N], Zbig[:, :N]
    bias = None if bb is None else _to_torch(bb, dtype)
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    cr.convrot_linear_ex(X, Wq, sw, g, bias, act, Y=Y, ws=ws, addend=Z)
    assert cr.convrot_read_device_status(ws) == 0
    torch.cuda.synchronize()
    # the padding columns of Y were not written
    assert torch.isnan(Ybig[:, N:]).all()
    rows = _rows_sample(M)
    wq_ref, sw_ref = oracle.prepare_weight(_to_f64(wb, dtype), g)
    ref = oracle.linear_ex(_to_f64(xb[rows], dtype), wq_ref, sw_ref, g, None if bb is None else _to_f64(bb, dtype),
                           addend=_to_f64(zb[rows], dtype), gelu=(act == GELU))
    y = _from_torch(Y.contiguous(), dtype)[rows]
    err = nrmse(y, ref)
    assert err <= NRMSE_TOL, f"{name}: NRMSE {err}"
    _check_elementwise(ws, M, K, rows, _to_f64(xb[rows], dtype), _to_f64(wb, dtype), g, TENSOR, Wq, sw, y,
                       None if bb is None else _to_f64(bb, dtype), _to_f64(zb[rows], dtype), act, dtype)


def test_strided_quant_act_is_the_dense_one(cr):
    import torch

    d = synth.make_workload("dit_qkv_1024")
    g = d["workload"].g
    X = _to_torch(d["x"], BF16)
    M, K = X.shape
    Xbig = torch.zeros((M, K + 136), dtype=X.dtype, device="cuda")
    Xbig[:, :K] = X
    q0, s0 = cr.convrot_quant_act(X, g)
    q1, s1 = cr.convrot_quant_act_ex(Xbig[:, :K], g)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and torch.equal(s0, s1)


@pytest.mark.parametrize("M", [200, 16])
def test_layer_wrapper_runs_the_variant_entry_points(cr, M):
    """ConvRotLinear with fp16, per-channel scales, GELU and an addend gives, bit for bit, what the
    direct calls it stands for give, and the default wrapper what convrot_linear gives."""
    import torch

    N, K, g = 264, 1024, 256
    rng = np.random.default_rng(M)
    x = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = synth.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = synth.f32_to_bf16_bits((rng.standard_normal(N) * 0.01).astype(np.float32))
    z = synth.f32_to_bf16_bits((rng.standard_normal((M, N)) * 0.05).astype(np.float32))
    X, W, B, Z = (_to_torch(_as_dtype_bits(t, F16), F16) for t in (x, w, b, z))

    layer = cr.ConvRotLinear(W, B, g, wscale_mode=cr.WSCALE_CHANNEL, activation=cr.ACT_GELU_ERF)
    assert layer.w_scale.shape == (N,)
    Y = layer(X, addend=Z)
    Wq, sw = cr.convrot_prepare_weight_ex(W, g, cr.WSCALE_CHANNEL)
    Y_direct = cr.convrot_linear_ex(X, Wq, sw, g, B, cr.ACT_GELU_ERF, addend=Z)
    torch.cuda.synchronize()
    assert torch.equal(layer.Wq, Wq) and torch.equal(layer.w_scale, sw)
    assert Y.dtype == torch.float16 and torch.equal(Y.view(torch.int16), Y_direct.view(torch.int16))

    Xb, Wb, Bb = (_to_torch(t, BF16) for t in (x, w, b))
    plain = cr.ConvRotLinear(Wb, Bb, g)
    Wq_b, sw_b = cr.convrot_prepare_weight(Wb, g)
    Y_plain = plain(Xb)
    torch.cuda.synchronize()
    assert torch.equal(Y_plain.view(torch.int16), cr.convrot_linear(Xb, Wq_b, sw_b, g, Bb).view(torch.int16))
