"""convrot_linear_noalloc, the entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a plugin inside an application that owns
the device-memory budget and hands over only input and output buffers, or a
latency-critical loop where an allocation could synchronise the device. This
entry point runs the same kernels as convrot_linear on a built-in scratch
array instead of a caller workspace. These tests call it through the C ABI and
compare it with convrot_linear, twice in a row with different layers, so a
result that depended on the previous call's scratch contents would show.
The file is collected last on purpose.
"""

from __future__ import annotations

import numpy as np
import pytest

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


def _call_both(cr, name):
    import torch

    L = cr.lib()
    d = synth.make_workload(name)
    w = d["workload"]
    M, K, N, g = w.M, w.K, w.N, w.g
    Wq, sw = cr.convrot_prepare_weight(to_torch_bf16(d["w"]), g)
    X = to_torch_bf16(d["x"])
    bias = None if d["bias"] is None else to_torch_bf16(d["bias"])
    stream = torch.cuda.current_stream().cuda_stream

    # the existing entry point, with a caller workspace
    ws = torch.empty(L.convrot_linear_workspace_bytes(M, N, K, g), dtype=torch.uint8, device="cuda")
    Y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = L.convrot_linear(X.data_ptr(), M, K, g, Wq.data_ptr(), sw.data_ptr(), N,
                          None if bias is None else bias.data_ptr(), Y_ref.data_ptr(), ws.data_ptr(), ws.numel(),
                          stream)
    assert st == 0

    # the allocation-free one
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    dev_status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = L.convrot_linear_noalloc(X.data_ptr(), M, K, g, Wq.data_ptr(), sw.data_ptr(), N,
                                  None if bias is None else bias.data_ptr(), Y.data_ptr(), dev_status.data_ptr(),
                                  stream)
    assert st == 0
    torch.cuda.synchronize()
    assert int(dev_status.item()) == 0
    err = nrmse(bf16_tensor_to_f64(Y), bf16_tensor_to_f64(Y_ref))
    assert err <= NRMSE_TOL
    # same kernels on the same inputs: the results are in fact identical
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))


def test_noalloc_matches_linear_on_two_calls_in_a_row(cr):
    _call_both(cr, "dit_qkv_1024")   # g = 256, with bias, 14.2 MB of codes in the scratch
    _call_both(cr, "textenc_m128")   # g = 128, no bias, a smaller call over the same scratch


def test_noalloc_rejects_calls_beyond_its_scratch(cr):
    L = cr.lib()
    fake = 0x10000  # never dereferenced: the size check comes first
    M, K, N = 16896, 12288, 3072   # 207 MB of codes > CONVROT_NOALLOC_SCRATCH_BYTES
    assert L.convrot_linear_workspace_bytes(M, N, K, 256) > 64 << 20
    st = L.convrot_linear_noalloc(fake, M, K, 256, fake, fake, N, None, fake, None, None)
    assert st == 3  # CONVROT_ERR_WORKSPACE
    # and a bad shape is still reported as such
    assert L.convrot_linear_noalloc(fake, 8, 300, 256, fake, fake, 256, None, fake, None, None) == 1
