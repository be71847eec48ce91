"""The measurement record the pair GEMM and the int8 probe leave in their workspace
(include/convrot.h, CONVROT_WS_CLOCK_RECORD_OFFSET): two (%clock64, %globaltimer)
readings of one thread, from which the SM clock of the launch follows."""

import pytest
import torch

import w8a8_rotated_int8_token_b200 as cr

pytestmark = pytest.mark.gpu

OFFSET = 64


def _record(ws):
    return ws[OFFSET:OFFSET + 32].view(torch.int64).tolist()


def _mhz(rec):
    return (rec[2] - rec[0]) / (rec[3] - rec[1]) * 1e3


def test_pair_gemm_writes_a_plausible_clock_record():
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    M, K, N = 1024, 3072, 4096
    W = (torch.randn((N, K), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    X = torch.randn((M, K), generator=g, device=dev).to(torch.bfloat16)
    Wq, sw = cr.convrot_prepare_weight(W, 256)
    ws = torch.zeros((cr.convrot_linear_workspace_bytes(M, N, K, 256),), dtype=torch.uint8, device=dev)
    cr.convrot_linear(X, Wq, sw, 256, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    rec = _record(ws)
    assert rec[2] > rec[0] > 0 and rec[3] > rec[1] > 0
    assert 200.0 < _mhz(rec) < 3000.0


def test_weight_streaming_gemm_leaves_the_record_untouched():
    dev = torch.device("cuda", 0)
    M, K, N = 16, 4096, 4096
    W = (torch.randn((N, K), device=dev) * 0.02).to(torch.bfloat16)
    X = torch.randn((M, K), device=dev).to(torch.bfloat16)
    Wq, sw = cr.convrot_prepare_weight(W, 128)
    ws = torch.zeros((cr.convrot_linear_workspace_bytes(M, N, K, 128),), dtype=torch.uint8, device=dev)
    ws[OFFSET:OFFSET + 32] = 7
    cr.convrot_linear(X, Wq, sw, 128, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    assert all(int(b) == 7 for b in ws[OFFSET:OFFSET + 32].tolist())


def test_probe_writes_a_plausible_clock_record():
    dev = torch.device("cuda", 0)
    ws = torch.zeros((256,), dtype=torch.uint8, device=dev)
    cr.convrot_probe_i8_peak(256, ws=ws)
    assert cr.convrot_read_device_status(ws) == 0
    rec = _record(ws)
    assert rec[2] > rec[0] > 0 and rec[3] > rec[1] > 0
    assert 200.0 < _mhz(rec) < 3000.0
