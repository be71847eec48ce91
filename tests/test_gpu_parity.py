"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

Small cases are compared element by element; the full-size workloads run in
the same launch configuration the benchmark times and are compared on sampled
token rows (rows are independent in every step of the method, so the oracle
run on a subset of rows gives exactly those rows' results).
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from parity import (NRMSE_TOL, bf16_tensor_to_f64, check_codes, check_output_elementwise, nrmse,
                    to_torch_bf16)
from test_abi import linear_ws_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cr():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_rotated_int8_token_b200 as cr

    cr.lib()  # loads libconvrot.so or raises
    return cr


def _rows_sample(M: int, n: int = 512, seed: int = 0) -> np.ndarray:
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    head = np.arange(128)
    tail = np.arange(M - 128, M)
    mid = rng.choice(np.arange(128, M - 128), n - 256, replace=False)
    return np.unique(np.concatenate([head, mid, tail]))


# ------------------------------------------------------------ rotate + quant


def _quant_case(cr, xbits: np.ndarray, g: int):
    import torch

    X = to_torch_bf16(xbits)
    Xq, s = cr.convrot_quant_act(X, g)
    torch.cuda.synchronize()
    x = oracle.bf16_to_f64(xbits)
    xr = oracle.rotate(x, g)
    q_ref, s_ref = oracle.quantize_per_token(xr)
    return check_codes(Xq.cpu().numpy(), s.cpu().numpy(), xr, q_ref, s_ref)


@pytest.mark.parametrize("name", ["tiny", "dit_qkv_1024", "textenc_m512"])
def test_quant_act_matches_oracle_on_workloads(cr, name):
    d = synth.make_workload(name)
    _quant_case(cr, d["x"], d["workload"].g)


@pytest.mark.parametrize("M,K,g", [(1, 256, 256), (3, 128, 128), (131, 384, 128), (130, 768, 256),
                                   (300, 12288, 256), (7, 32768, 256), (5, 32768, 128)])
def test_quant_act_ragged_and_extreme_shapes(cr, M, K, g):
    rng = np.random.default_rng(M * 7919 + K + g)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, max(1, K // 100), replace=False)] *= 50.0
    _quant_case(cr, synth.f32_to_bf16_bits(x), g)


@pytest.mark.parametrize("g", [128, 256])
def test_quant_act_special_rows(cr, g):
    K = 4 * g
    rng = np.random.default_rng(3)
    rows = [np.zeros(K, np.float32)]                        # zero token: scale 0, codes 0
    spike = np.zeros(K, np.float32); spike[g + 37] = -3.0   # one channel: a full +-127 group
    rows.append(spike)
    const = np.zeros(K, np.float32); const[2 * g:3 * g] = 0.75  # constant group: (127, 0, ...)
    rows.append(const)
    rows.append((rng.standard_normal(K) * 1e-34).astype(np.float32))  # tiny token (scale near 2^-120)
    rows.append((rng.standard_normal(K) * 1e-30).astype(np.float32))  # tiny token
    rows.append((rng.standard_normal(K) * 1e33).astype(np.float32))   # huge token
    rows.append(np.full(K, -2.0, np.float32))
    xbits = synth.f32_to_bf16_bits(np.stack(rows))
    _quant_case(cr, xbits, g)
    import torch

    Xq, s = cr.convrot_quant_act(to_torch_bf16(xbits), g)
    Xq = Xq.cpu().numpy()
    assert float(s[0]) == 0.0 and not Xq[0].any()
    h = oracle.hadamard(g)
    assert np.array_equal(Xq[1, g:2 * g].astype(np.int32), -127 * h[37].astype(np.int32))
    assert not Xq[1, :g].any() and not Xq[1, 2 * g:].any()
    expect = np.zeros(K, np.int8); expect[2 * g] = 127
    assert np.array_equal(Xq[2], expect)
    torch.cuda.synchronize()


def test_quant_act_scale_equivariance_and_symmetry(cr):
    import torch

    d = synth.make_workload("tiny")
    x = synth.bf16_bits_to_f32(d["x"])
    q0, s0 = cr.convrot_quant_act(to_torch_bf16(d["x"]), 256)
    q1, s1 = cr.convrot_quant_act(to_torch_bf16(synth.f32_to_bf16_bits(x * 8.0)), 256)
    q2, s2 = cr.convrot_quant_act(to_torch_bf16(synth.f32_to_bf16_bits(-x)), 256)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and torch.equal(s1, s0 * 8.0)
    assert torch.equal(q2, -q0) and torch.equal(s2, s0)


# -------------------------------------------------------------- weights


@pytest.mark.parametrize("name", ["tiny", "dit_qkv_1024", "textenc_m16"])
def test_prepare_weight_matches_oracle(cr, name):
    import torch

    d = synth.make_workload(name)
    g = d["workload"].g
    W = to_torch_bf16(d["w"])
    Wq, sw = cr.convrot_prepare_weight(W, g)
    torch.cuda.synchronize()
    w = oracle.bf16_to_f64(d["w"])
    wr = oracle.rotate(w, g)
    q_ref, s_ref = oracle.quantize_tensorwise(wr)
    check_codes(Wq.cpu().numpy(), sw.cpu().numpy(), wr, q_ref, np.array([s_ref]), per_token=False)
    assert int(np.abs(Wq.cpu().numpy().astype(np.int32)).max()) == 127


# ---------------------------------------------------------- int32 GEMM


def _gemm_exact(cr, xq: np.ndarray, wq: np.ndarray, rows=None):
    import torch

    acc = cr.convrot_gemm_s32(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda())
    torch.cuda.synchronize()
    acc = acc.cpu().numpy()
    if rows is None:
        ref = oracle.gemm_s32(xq, wq)
        assert np.array_equal(acc, ref)
    else:
        ref = oracle.gemm_s32(xq[rows], wq)
        assert np.array_equal(acc[rows], ref)


@pytest.mark.parametrize("M,N,K", [(64, 256, 256), (1, 8, 16), (1, 256, 128), (130, 264, 272), (257, 520, 4096),
                                   (128, 1024, 12288), (513, 12288, 128),
                                   (8, 20480, 256)])  # weight-streaming form, 160 tiles: two per CTA on some SMs
def test_gemm_s32_bit_exact(cr, M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    _gemm_exact(cr, xq, wq)


def test_gemm_s32_extreme_accumulators(cr):
    K = 12288  # |acc| up to K * 127^2 = 198,193,152
    xq = np.full((130, K), 127, np.int8)
    xq[1::2] = -127
    wq = np.full((264, K), 127, np.int8)
    wq[::3] = -127
    wq[5, ::2] = -127
    _gemm_exact(cr, xq, wq)


def test_gemm_s32_full_size_sampled(cr):
    d = synth.make_workload("dit_qkv_1024")
    g = d["workload"].g
    xq, _ = oracle.quant_act(oracle.bf16_to_f64(d["x"]), g)
    wq, _ = oracle.prepare_weight(oracle.bf16_to_f64(d["w"]), g)
    _gemm_exact(cr, xq, wq, rows=_rows_sample(xq.shape[0]))


def test_gemm_dequant_on_identical_codes(cr):
    import torch

    d = synth.make_workload("dit_qkv_1024")
    g = d["workload"].g
    x = oracle.bf16_to_f64(d["x"])
    xq, sx = oracle.quant_act(x, g)
    wq, sw = oracle.prepare_weight(oracle.bf16_to_f64(d["w"]), g)
    bias = d["bias"]
    Y = cr.convrot_gemm_dequant(torch.from_numpy(xq).cuda(), torch.from_numpy(sx).cuda(),
                                torch.from_numpy(wq).cuda(), torch.tensor([sw], dtype=torch.float32).cuda(),
                                to_torch_bf16(bias))
    torch.cuda.synchronize()
    rows = _rows_sample(xq.shape[0])
    y = bf16_tensor_to_f64(Y)[rows]
    ref = oracle.dequant(oracle.gemm_s32(xq[rows], wq), sx[rows], sw, oracle.bf16_to_f64(bias))
    # same codes, so only float32 dequant rounding and the bf16 rounding remain
    err = np.abs(y - ref)
    assert np.all(err <= 2.0**-8 * np.abs(ref) + 1e-6 * np.abs(ref).max())
    assert nrmse(y, ref) < 2e-3


# ------------------------------------------------------------ end to end


def _linear_case(cr, d, rows=None, one_launch=False):
    import torch

    w = d["workload"]
    g = w.g
    W = to_torch_bf16(d["w"])
    Wq, sw = cr.convrot_prepare_weight(W, g)
    bias = None if d["bias"] is None else to_torch_bf16(d["bias"])
    X = to_torch_bf16(d["x"])
    M, K = d["x"].shape
    N = d["w"].shape[0]
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    layer = cr.convrot_linear_one_launch if one_launch else cr.convrot_linear
    Y = layer(X, Wq, sw, g, bias, ws=ws)
    status = cr.convrot_read_device_status(ws)
    assert status == 0
    if rows is None:
        rows = np.arange(M)
    xs = oracle.bf16_to_f64(d["x"][rows])
    wq_ref, sw_ref = oracle.prepare_weight(oracle.bf16_to_f64(d["w"]), g)
    b = None if d["bias"] is None else oracle.bf16_to_f64(d["bias"])
    ref = oracle.linear(xs, wq_ref, sw_ref, g, b)
    y = bf16_tensor_to_f64(Y)[rows]
    err = nrmse(y, ref)
    assert err <= NRMSE_TOL, f"{w.name}: NRMSE {err}"
    # the codes and token scales this call left in its workspace
    wsn = ws.cpu().numpy()
    lay = linear_ws_layout(M, K)
    sx_gpu = wsn[lay["scale"]:lay["scale"] + 4 * M].view(np.float32)[rows]
    xq_gpu = wsn[lay["codes"]:lay["codes"] + M * K].view(np.int8).reshape(M, K)[rows]
    xr = oracle.rotate(xs, g)
    q_ref, s_ref = oracle.quantize_per_token(xr)
    check_codes(xq_gpu, sx_gpu, xr, q_ref, s_ref)
    # the weight codes and scale the kernel prepared, then every output element
    # against the oracle's arithmetic on the kernel's own codes and scales
    wq_gpu = Wq.cpu().numpy()
    sw_gpu = sw.cpu().numpy().reshape(1)
    check_codes(wq_gpu, sw_gpu, oracle.rotate(oracle.bf16_to_f64(d["w"]), g), wq_ref, np.array([sw_ref]),
                per_token=False)
    check_output_elementwise(y, oracle.gemm_s32(xq_gpu, wq_gpu), sx_gpu, float(sw_gpu[0]), b)
    return Y, err


@pytest.mark.parametrize("name", ["tiny", "dit_qkv_1024", "dit_mlp_up_1024", "textenc_m1", "textenc_m16",
                                  "textenc_m128", "textenc_m512"])
def test_linear_matches_oracle(cr, name):
    d = synth.make_workload(name)
    _linear_case(cr, d, rows=_rows_sample(d["x"].shape[0]))


def test_linear_matches_oracle_mlp_2048(cr):
    d = synth.make_workload("dit_mlp_2048")
    _linear_case(cr, d, rows=_rows_sample(d["x"].shape[0], 384))


def test_linear_matches_oracle_mlp_down_1024(cr):
    up = synth.make_workload("dit_mlp_up_1024")
    g = up["workload"].g
    wq, sw = oracle.prepare_weight(oracle.bf16_to_f64(up["w"]), g)
    y_up = oracle.linear(oracle.bf16_to_f64(up["x"]), wq, sw, g)  # the oracle's up output feeds both sides
    dn = synth.make_workload("dit_mlp_down_1024", x_up_output=y_up)
    _linear_case(cr, dn, rows=_rows_sample(dn["x"].shape[0], 256))


def test_linear_is_deterministic(cr):
    import torch

    d = synth.make_workload("dit_qkv_1024")
    Y1, _ = _linear_case(cr, d, rows=np.arange(64))
    Y2, _ = _linear_case(cr, d, rows=np.arange(64))
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_zero_input_gives_zero_output_and_bias(cr):
    import torch

    d = synth.make_workload("dit_qkv_1024")
    W = to_torch_bf16(d["w"])
    Wq, sw = cr.convrot_prepare_weight(W, 256)
    X = torch.zeros((130, 3072), dtype=torch.bfloat16, device="cuda")
    Y = cr.convrot_linear(X, Wq, sw, 256)
    assert not Y.view(torch.int16).any()
    b = to_torch_bf16(d["bias"])
    Yb = cr.convrot_linear(X, Wq, sw, 256, b)
    torch.cuda.synchronize()
    assert torch.equal(Yb.view(torch.int16), b.view(torch.int16).expand(130, -1))


def test_empty_batch_gives_empty_output(cr):
    """M = 0 (no tokens) through every public entry point: empty results, no launch, no error,
    and the next call on the same workspace still matches the oracle."""
    import torch

    M, N, K, g = 0, 264, 1024, 256
    d = _random_layer(130, N, K, g)
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(d["w"]), g)
    X0 = torch.empty((0, K), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(cr.convrot_linear_workspace_bytes(130, N, K, g), dtype=torch.uint8, device="cuda")
    ws.view(torch.int32)[0] = 5  # a status word left by an earlier call (the timeout code)
    assert cr.convrot_linear(X0, Wq, sw, g, ws=ws).shape == (0, N)
    assert cr.convrot_linear_one_launch(X0, Wq, sw, g, ws=ws).shape == (0, N)
    Xq0, s0 = cr.convrot_quant_act(X0, g)
    assert Xq0.shape == (0, K) and s0.shape == (0,)
    Wc, swc = cr.convrot_prepare_weight_ex(to_torch_bf16(d["w"]).half(), g, cr.WSCALE_CHANNEL)
    assert cr.convrot_linear_ex(X0.half(), Wc, swc, g, activation=cr.ACT_GELU_ERF).shape == (0, N)
    assert cr.convrot_gemm_dequant(Xq0, s0, Wq, sw).shape == (0, N)
    assert cr.convrot_gemm_s32(Xq0, Wq).shape == (0, N)
    layer = cr.ConvRotLinear(to_torch_bf16(d["w"]), None, g)
    assert layer(X0).shape == (0, N)
    # the allocation-free entry reports this call's status (0), not a leftover value
    L = cr.lib()
    dev_status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert L.convrot_linear_noalloc(None, 0, K, g, Wq.data_ptr(), sw.data_ptr(), N, None, None,
                                    dev_status.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(dev_status.item()) == 0
    assert cr.convrot_read_device_status(ws) == 5  # the empty calls left the workspace as it was
    # a full call on the same workspace: its first kernel resets the status word
    Y = cr.convrot_linear(to_torch_bf16(d["x"]), Wq, sw, g, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    wq_ref, sw_ref = oracle.prepare_weight(oracle.bf16_to_f64(d["w"]), g)
    ref = oracle.linear(oracle.bf16_to_f64(d["x"]), wq_ref, sw_ref, g, None)
    assert nrmse(bf16_tensor_to_f64(Y), ref) <= NRMSE_TOL


def _random_layer(M, N, K, g):
    rng = np.random.default_rng(M + N + K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, max(1, K // 100), replace=False)] *= 50.0
    return {"workload": type("W", (), {"name": f"{M}x{K}x{N}", "g": g})(),
            "x": synth.f32_to_bf16_bits(x),
            "w": synth.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32)),
            "bias": synth.f32_to_bf16_bits((rng.standard_normal(N) * 0.01).astype(np.float32))}


@pytest.mark.parametrize("M,N,K,g", [(130, 264, 20480, 256), (129, 136, 20608, 128),
                                     (67, 264, 32768, 256),    # largest K
                                     (1, 16, 384, 128), (385, 520, 1024, 256),
                                     (33, 19712, 512, 256)])  # 154 weight tiles at M <= 64 (vocabulary-sized N)
def test_linear_ragged_and_large_k(cr, M, N, K, g):
    _linear_case(cr, _random_layer(M, N, K, g))


# The weight-streaming GEMM (M <= 64) split over all SMs: (weight tile, k-block)
# units in equal contiguous ranges per CTA, partial tiles summed by the last CTA
# to arrive. Cases: tiles shared by two and three CTAs (K = 12288: 96 k-blocks
# per tile), one k-block per tile (every unit a whole tile), fewer units than
# SMs, N not a multiple of 128 (the last tile's rows past N), M at 1, 17 and 64
# (16-, 32- and 64-token MMA columns), and more tiles than SMs.
@pytest.mark.parametrize("M,N,K,g", [(1, 12288, 4096, 128), (17, 1032, 12288, 256), (64, 384, 12288, 256),
                                     (5, 8192, 128, 128), (3, 200, 256, 256), (40, 2056, 768, 256),
                                     (9, 40960, 1024, 256)])
def test_linear_weight_streaming_split(cr, M, N, K, g):
    _linear_case(cr, _random_layer(M, N, K, g))


def test_linear_weight_streaming_split_is_deterministic(cr):
    # the partial sums meet in whatever order the CTAs arrive; integer sums make the
    # result independent of it, so repeated calls give identical bits
    import torch

    d = _random_layer(16, 12288, 4096, 128)
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(d["w"]), 128)
    X = to_torch_bf16(d["x"])
    outs = [cr.convrot_linear(X, Wq, sw, 128, to_torch_bf16(d["bias"])) for _ in range(4)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


# For a few tokens (M * K <= 16384) convrot_linear is one kernel that rotates
# and quantises the tokens into shared memory itself: the same arithmetic in
# the same order as the rotate+quantise kernel, so its codes, scales and
# output equal those of the two halves (convrot_quant_act, then
# convrot_gemm_dequant on the weight-streaming GEMM) bit for bit. Cases: the
# text-encoder layer at 1 and 4 tokens, K at its limit (8192, two ring
# stages), 16 tokens, more weight tiles than SMs, the smallest K, N not a
# multiple of the tile rows, both g, a zero token among others.
@pytest.mark.parametrize("M,N,K,g", [(1, 12288, 4096, 128), (4, 12288, 4096, 128), (2, 1032, 8192, 256),
                                     (1, 4104, 8192, 128), (16, 19712, 1024, 256), (16, 8, 128, 128),
                                     (7, 264, 256, 256), (11, 2056, 768, 256)])
def test_linear_one_kernel_form_equals_the_two_halves(cr, M, N, K, g):
    import torch

    assert cr.lib().convrot_linear_launch_count(M, N, K, g) == 1
    d = _random_layer(M, N, K, g)
    if M > 2:
        d["x"][M // 2] = 0  # an all-zero token: scale 0, codes 0
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(d["w"]), g)
    X = to_torch_bf16(d["x"])
    bias = to_torch_bf16(d["bias"])
    ws = torch.zeros(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    Y = cr.convrot_linear(X, Wq, sw, g, bias, ws=ws)
    Xq, sx = cr.convrot_quant_act(X, g)
    Y2 = cr.convrot_gemm_dequant(Xq, sx, Wq, sw, bias)
    torch.cuda.synchronize()
    assert cr.convrot_read_device_status(ws) == 0
    wsn = ws.cpu().numpy()
    lay = linear_ws_layout(M, K)
    sx_ws = wsn[lay["scale"]:lay["scale"] + 4 * M].view(np.float32)
    xq_ws = wsn[lay["codes"]:lay["codes"] + M * K].view(np.int8).reshape(M, K)
    assert np.array_equal(xq_ws, Xq.cpu().numpy())
    assert np.array_equal(sx_ws.view(np.uint32), sx.cpu().numpy().view(np.uint32))
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    # and the oracle: near-tie codes only, every output element within its bound
    ref = oracle.linear(oracle.bf16_to_f64(d["x"]), *oracle.prepare_weight(oracle.bf16_to_f64(d["w"]), g), g,
                        oracle.bf16_to_f64(d["bias"]))
    assert nrmse(bf16_tensor_to_f64(Y), ref) <= NRMSE_TOL


def test_linear_one_kernel_form_back_to_back_on_rotating_buffers(cr):
    # calls that overlap through programmatic launch: each one's weight stream
    # starts while the previous call runs; every output must match its own
    # two-halves result
    import torch

    M, N, K, g = 4, 12288, 4096, 128
    layers = []
    for i in range(3):
        d = _random_layer(M + i - 2, N, K, g)
        Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(d["w"]), g)
        X = to_torch_bf16(d["x"])
        layers.append((X, Wq, sw, cr.convrot_gemm_dequant(*cr.convrot_quant_act(X, g), Wq, sw)))
    torch.cuda.synchronize()
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    outs = []
    for r in range(12):
        X, Wq, sw, _ = layers[r % 3]
        outs.append((r % 3, cr.convrot_linear(X, Wq, sw, g, ws=ws)))
    torch.cuda.synchronize()
    assert cr.convrot_read_device_status(ws) == 0
    for i, y in outs:
        assert torch.equal(y.view(torch.int16), layers[i][3].view(torch.int16))


@pytest.mark.parametrize("M,N,K,g", [(130, 264, 20480, 256),   # largest K of the one-launch form
                                     (1, 16, 384, 128), (385, 520, 1024, 256), (64, 256, 256, 256)])
def test_linear_one_launch_matches_oracle(cr, M, N, K, g):
    _linear_case(cr, _random_layer(M, N, K, g), one_launch=True)


def test_linear_one_launch_on_the_bench_layer(cr):
    d = synth.make_workload("dit_qkv_1024")
    _linear_case(cr, d, rows=_rows_sample(d["x"].shape[0]), one_launch=True)


def test_linear_one_launch_rejects_k_beyond_its_workers(cr):
    import torch

    M, N, K = 64, 256, 20608
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    sw = torch.ones((1,), dtype=torch.float32, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_linear_one_launch(X, Wq, sw, 128)
    assert e.value.status == 2


@pytest.mark.parametrize("one_launch", [False, True])
def test_linear_back_to_back_calls_on_one_workspace(cr, one_launch):
    """Consecutive calls reuse the workspace: later calls must not see earlier readiness counters."""
    import torch

    a = synth.make_workload("dit_qkv_1024")
    b = synth.make_workload("tiny")
    Wa, sa = cr.convrot_prepare_weight(to_torch_bf16(a["w"]), 256)
    Wb, sb = cr.convrot_prepare_weight(to_torch_bf16(b["w"]), 256)
    ws = torch.empty(cr.convrot_linear_workspace_bytes(4608, 9216, 3072, 256), dtype=torch.uint8, device="cuda")
    Xa = to_torch_bf16(a["x"])
    Xb = to_torch_bf16(b["x"])
    ref_a = cr.convrot_linear(Xa, Wa, sa, 256, to_torch_bf16(a["bias"]))
    ref_b = cr.convrot_linear(Xb, Wb, sb, 256)
    outs = []
    layer = cr.convrot_linear_one_launch if one_launch else cr.convrot_linear
    if one_launch:  # the same form on both sides of the comparison
        ref_a = layer(Xa, Wa, sa, 256, to_torch_bf16(a["bias"]))
        ref_b = layer(Xb, Wb, sb, 256)
    for i in range(6):  # alternate layers on the same workspace, no synchronisation in between
        if i % 2 == 0:
            outs.append(("a", layer(Xa, Wa, sa, 256, to_torch_bf16(a["bias"]), ws=ws)))
        else:
            outs.append(("b", layer(Xb, Wb, sb, 256, ws=ws)))
    torch.cuda.synchronize()
    assert cr.convrot_read_device_status(ws) == 0
    for tag, y in outs:
        ref = ref_a if tag == "a" else ref_b
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("M,N,K", [(130, 264, 256), (1, 8, 128), (257, 1032, 384)])
def test_linear_writes_only_its_output(cr, M, N, K):
    import torch

    g = 128 if K % 256 else 256
    rng = np.random.default_rng(M + N)
    x = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    w = synth.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(w), g)
    guard = 4096
    sentinel = 0x5A5A
    buf = torch.full((guard + M * N + guard,), sentinel, dtype=torch.int16, device="cuda")
    Y = buf[guard:guard + M * N].view(torch.bfloat16).view(M, N)
    cr.convrot_linear(to_torch_bf16(x), Wq, sw, g, Y=Y)
    torch.cuda.synchronize()
    assert bool((buf[:guard] == sentinel).all()) and bool((buf[guard + M * N:] == sentinel).all())
    ref = oracle.linear(oracle.bf16_to_f64(x), *oracle.prepare_weight(oracle.bf16_to_f64(w), g), g)
    assert nrmse(bf16_tensor_to_f64(Y), ref) <= NRMSE_TOL


def test_bounded_wait_reports_timeout_without_fault(cr):
    import torch

    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    cr.convrot_test_wait_timeout(ws, 5_000_000)  # 5 ms; nothing will complete the barrier
    assert cr.convrot_read_device_status(ws) == 5
    # the context is still usable and a normal call clears the word
    d = synth.make_workload("tiny")
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(d["w"]), 256)
    ws2 = torch.empty(cr.convrot_linear_workspace_bytes(64, 256, 256, 256), dtype=torch.uint8, device="cuda")
    ws2[:4] = 5
    cr.convrot_linear(to_torch_bf16(d["x"]), Wq, sw, 256, ws=ws2)
    assert cr.convrot_read_device_status(ws2) == 0
