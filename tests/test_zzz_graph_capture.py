"""The layer inside a CUDA graph (stream capture), on a B200.

A caller that replays a captured graph copies each new input into the captured
buffer and replays. These tests capture convrot_linear on both GEMM forms (CTA
pairs for M > 64, weight streaming for M <= 64), replay it on different inputs
and compare each output bit for bit with an eager call on the same input (the
parity tests compare those with the oracle), and the last one with the oracle
as well. convrot_linear_one_launch must refuse a capturing stream: its
per-call tag is drawn on the host and a replay would reuse it.

Collected last: a capture that went wrong could leave the process's CUDA state
unusable for the tests after it.
"""

from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from parity import NRMSE_TOL, bf16_tensor_to_f64, nrmse, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cr():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_rotated_int8_token_b200 as cr

    cr.lib()
    return cr


def _layer(M, N, K, seed):
    """Two activations (with outlier channels), a weight and a bias, as bf16 bits."""
    rng = np.random.default_rng(seed)

    def act():
        a = rng.standard_normal((M, K)).astype(np.float32)
        a[:, rng.choice(K, max(1, K // 100), replace=False)] *= 50.0
        return synth.f32_to_bf16_bits(a)

    x1, x2 = act(), act()
    w = synth.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = synth.f32_to_bf16_bits((rng.standard_normal(N) * 0.01).astype(np.float32))
    return x1, x2, w, b


def _warm_up(cr, X, Wq, sw, g, bias, Y, ws):
    """One eager call on a side stream before capturing (the usual order for a graph)."""
    import torch

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        cr.convrot_linear(X, Wq, sw, g, bias, Y=Y, ws=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()


@pytest.mark.parametrize("M,N,K,g", [(576, 1024, 3072, 256),   # CTA-pair GEMM, ragged last M tile
                                     (16, 2048, 4096, 128),    # weight-streaming GEMM
                                     (2, 12288, 4096, 128)])   # the one-kernel form (M * K <= 16384)
def test_captured_linear_replays_on_new_inputs(cr, M, N, K, g):
    import torch

    x1, x2, wb, bb = _layer(M, N, K, seed=M + N)
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(wb), g)
    bias = to_torch_bf16(bb)
    X1, X2 = to_torch_bf16(x1), to_torch_bf16(x2)
    Y1 = cr.convrot_linear(X1, Wq, sw, g, bias)
    Y2 = cr.convrot_linear(X2, Wq, sw, g, bias)

    Xs = X1.clone()
    Ys = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    _warm_up(cr, Xs, Wq, sw, g, bias, Ys, ws)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cr.convrot_linear(Xs, Wq, sw, g, bias, Y=Ys, ws=ws)

    for X, Y_eager in ((X2, Y2), (X1, Y1), (X2, Y2)):
        Ys.fill_(float("nan"))
        Xs.copy_(X)
        graph.replay()
        torch.cuda.synchronize()
        assert cr.convrot_read_device_status(ws) == 0
        assert torch.equal(Ys.view(torch.int16), Y_eager.view(torch.int16))

    wq_ref, sw_ref = oracle.prepare_weight(oracle.bf16_to_f64(wb), g)
    ref = oracle.linear(oracle.bf16_to_f64(x2), wq_ref, sw_ref, g, oracle.bf16_to_f64(bb))
    assert nrmse(bf16_tensor_to_f64(Ys), ref) <= NRMSE_TOL
    del graph


def test_one_launch_refuses_a_capturing_stream(cr):
    import torch

    M, N, K, g = 256, 512, 1024, 256
    x1, _, wb, _ = _layer(M, N, K, seed=7)
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(wb), g)
    X = to_torch_bf16(x1)
    Y_eager = cr.convrot_linear(X, Wq, sw, g)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(cr.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    _warm_up(cr, X, Wq, sw, g, None, Y, ws)
    L = cr.lib()
    graph = torch.cuda.CUDAGraph()
    statuses = []
    with torch.cuda.graph(graph):
        stream = torch.cuda.current_stream().cuda_stream
        statuses.append(L.convrot_linear_one_launch(X.data_ptr(), M, K, g, Wq.data_ptr(), sw.data_ptr(), N, None,
                                                    Y.data_ptr(), ws.data_ptr(), ws.numel(), stream))
        cr.convrot_linear(X, Wq, sw, g, Y=Y, ws=ws)  # the two-kernel form captures in the same graph
    assert statuses == [2]  # CONVROT_ERR_UNSUPPORTED, nothing enqueued
    Y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y_eager.view(torch.int16))
    del graph
    # outside a capture the one-launch form runs as usual
    Y1 = cr.convrot_linear_one_launch(X, Wq, sw, g, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    wq_ref, sw_ref = oracle.prepare_weight(oracle.bf16_to_f64(wb), g)
    ref = oracle.linear(oracle.bf16_to_f64(x1), wq_ref, sw_ref, g, None)
    assert nrmse(bf16_tensor_to_f64(Y1), ref) <= NRMSE_TOL
