"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before touching the GPU."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from w8a8_rotated_int8_token_b200 import build, _lib

    build.build()
    return _lib.load()


def _declared_entry_points():
    with open(os.path.join(ROOT, "include", "convrot.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"CONVROT_API\s+[\w\s\*]+?\b(convrot_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_entry_points()
    for required in ("convrot_prepare_weight", "convrot_quant_act", "convrot_linear",
                     "convrot_linear_workspace_bytes", "convrot_gemm_s32", "convrot_read_device_status",
                     "convrot_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    from w8a8_rotated_int8_token_b200 import _lib

    for name in _declared_entry_points():
        assert hasattr(L, name), name
        assert name in _lib.SIGNATURES, f"{name} has no ctypes signature"


def test_library_exports_nothing_else():
    import subprocess

    from w8a8_rotated_int8_token_b200 import _lib

    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(_declared_entry_points())


def linear_ws_layout(M, K, N=None):
    """Byte layout of convrot_linear's workspace, as include/convrot.h describes it
    (the split buffers of the weight-streaming GEMM, for 1 <= M <= 64 and at most 64 weight
    tiles of 128 rows, when N is given)."""
    up = lambda v, a: (v + a - 1) // a * a  # noqa: E731
    ready = 256
    scale = up(ready + 8 * ((M + 127) // 128), 256)
    codes = up(scale + 4 * M, 1024)
    total = up(codes + M * K, 256)
    lay = {"ready": ready, "scale": scale, "codes": codes, "total": total}
    if N is not None and 1 <= M <= 64 and (N + 127) // 128 <= 64:
        bnt = 16 if M <= 16 else (32 if M <= 32 else 64)
        lay["split_count"] = total
        lay["split_part"] = up(total + 4 * ((N + 127) // 128), 1024)
        lay["total"] = up(lay["split_part"] + 2 * 160 * bnt * 128 * 4, 256)
    return lay


def test_status_strings_and_version(L):
    assert L.convrot_abi_version() == 9
    for code in range(6):
        s = L.convrot_status_string(code)
        assert s and s != b"unknown status"
    assert L.convrot_status_string(99) == b"unknown status"


def test_workspace_sizes(L):
    # [status 256 B | ready counters 8 B per 128 tokens | scales 4M | codes M*K]
    M, N, K = 4608, 9216, 3072
    need = L.convrot_linear_workspace_bytes(M, N, K, 256)
    assert need == linear_ws_layout(M, K, N)["total"]
    assert need >= M * K + 4 * M + 8 * (M // 128) + 256
    assert L.convrot_linear_workspace_bytes(M, N, K, 64) == 0       # unsupported g
    assert L.convrot_linear_workspace_bytes(M, N, 3000, 256) == 0   # K % g != 0
    assert L.convrot_linear_workspace_bytes(M, 9212, K, 256) == 0   # N % 8 != 0
    assert L.convrot_linear_workspace_bytes(0, N, K, 256) == linear_ws_layout(0, K, N)["total"]  # M = 0 is valid
    # the weight-streaming GEMM's split buffers (M <= 64)
    for m in (1, 16, 17, 33, 64, 65):
        for n in (12288, 4096, 8192, 8200):
            assert L.convrot_linear_workspace_bytes(m, n, 4096, 128) == linear_ws_layout(m, 4096, n)["total"]
    assert L.convrot_linear_workspace_bytes(-1, N, K, 256) == 0
    assert L.convrot_gemm_workspace_bytes() == 256
    assert L.convrot_prepare_weight_workspace_bytes() >= 4


FAKE = 0x10000  # 16-byte aligned non-null value; never dereferenced: every call below fails validation


@pytest.mark.parametrize("args,expect", [
    # (X, M, K, g, Wq, w_scale, N, bias, Y, ws, ws_bytes)
    ((FAKE, 64, 256, 64, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 30), 2),      # g unsupported
    ((FAKE, 64, 300, 256, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 30), 1),     # K % g
    ((FAKE, 64, 65536, 256, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 40), 2),   # K above limit
    ((FAKE, 64, 256, 256, FAKE, FAKE, 0, None, FAKE, FAKE, 1 << 30), 1),       # N = 0
    ((FAKE, 64, 256, 256, FAKE, FAKE, 260, None, FAKE, FAKE, 1 << 30), 1),     # N % 8
    ((None, 64, 256, 256, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 30), 1),     # null X
    ((FAKE, 64, 256, 256, None, FAKE, 256, None, FAKE, FAKE, 1 << 30), 1),     # null Wq
    ((FAKE, 64, 256, 256, FAKE, None, 256, None, FAKE, FAKE, 1 << 30), 1),     # null w_scale
    ((FAKE, 64, 256, 256, FAKE, FAKE, 256, None, None, FAKE, 1 << 30), 1),     # null Y
    ((FAKE + 2, 64, 256, 256, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 30), 1),  # misaligned X
    ((FAKE, 64, 256, 256, FAKE, FAKE, 256, FAKE + 8, FAKE, FAKE, 1 << 30), 1),  # misaligned bias
    ((FAKE, 64, 256, 256, FAKE, FAKE, 256, None, FAKE, None, 1 << 30), 3),     # null workspace
    ((FAKE, 64, 256, 256, FAKE, FAKE, 256, None, FAKE, FAKE + 16, 1 << 30), 3),  # misaligned workspace
    ((FAKE, 64, 256, 256, FAKE, FAKE, 256, None, FAKE, FAKE, 100), 3),         # workspace too small
])
def test_linear_rejects_bad_arguments_on_host(L, args, expect):
    assert L.convrot_linear(*args, None) == expect


def test_other_entry_points_reject_bad_arguments_on_host(L):
    assert L.convrot_quant_act(FAKE, 8, 256, 512, FAKE, FAKE, None) == 2
    assert L.convrot_quant_act(None, 8, 256, 256, FAKE, FAKE, None) == 1
    assert L.convrot_quant_act(FAKE, 8, 256, 256, FAKE, FAKE + 2, None) == 1
    assert L.convrot_prepare_weight(FAKE, 8, 384, 256, FAKE, FAKE, FAKE, 256, None) == 1
    assert L.convrot_prepare_weight(FAKE, 8, 256, 256, FAKE, FAKE, FAKE, 2, None) == 3
    assert L.convrot_gemm_s32(FAKE, FAKE, 8, 6, 256, FAKE, FAKE, 256, None) == 1    # N % 4
    assert L.convrot_gemm_s32(FAKE, FAKE, 8, 8, 24, FAKE, FAKE, 256, None) == 1     # K % 16
    # more output tiles than an int counts (no such output fits in memory, but it must not wrap)
    assert L.convrot_gemm_s32(FAKE, FAKE, 2**31 - 1, 2**31 - 8, 256, FAKE, FAKE, 256, None) == 2
    assert L.convrot_gemm_s32(FAKE, FAKE, 8, 8, 256, FAKE, FAKE, 16, None) == 3     # workspace
    assert L.convrot_gemm_dequant(FAKE, None, FAKE, FAKE, 8, 8, 256, None, FAKE, FAKE, 256, None) == 1
    assert L.convrot_read_device_status(None, None) == 3
    assert L.convrot_test_wait_timeout(FAKE, 256, 10, None) == 1
    assert L.convrot_test_wait_timeout(FAKE, 256, 10**10, None) == 1
    # the timed variant needs both events
    assert L.convrot_linear_timed(FAKE, 64, 256, 256, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 30, None, None,
                                  FAKE, None) == 1
    assert L.convrot_linear_launch_count(4608, 9216, 3072, 256) == 2
    # a few tokens (M * K <= 16384, M <= 16, K <= 8192): one kernel
    assert L.convrot_linear_launch_count(1, 12288, 4096, 128) == 1
    assert L.convrot_linear_launch_count(4, 12288, 4096, 128) == 1
    assert L.convrot_linear_launch_count(2, 12288, 8192, 256) == 1
    assert L.convrot_linear_launch_count(16, 12288, 1024, 256) == 1
    assert L.convrot_linear_launch_count(5, 12288, 4096, 128) == 2
    assert L.convrot_linear_launch_count(17, 12288, 512, 256) == 2
    assert L.convrot_linear_launch_count(1, 12288, 8448, 256) == 2
    # the one-launch form: K beyond what one CTA's worker warps hold
    assert L.convrot_linear_one_launch(FAKE, 64, 20608, 128, FAKE, FAKE, 256, None, FAKE, FAKE, 1 << 40, None) == 2
    assert L.convrot_linear_one_launch(FAKE, 64, 256, 256, FAKE, FAKE, 256, None, None, FAKE, 1 << 30, None) == 1
    assert L.convrot_linear_launch_count(4608, 9216, 3000, 256) == 0


def test_variant_entry_points_reject_bad_arguments_on_host(L):
    # convrot_linear_ex(X, dtype, M, K, ldx, g, Wq, w_scale, wscale_mode, N, bias, addend, activation, Y, ldy,
    #                   ws, ws_bytes, stream)
    names = ["X", "dtype", "M", "K", "ldx", "g", "Wq", "w_scale", "mode", "N", "bias", "addend", "act", "Y", "ldy",
             "ws", "ws_bytes", "s"]
    ok = [FAKE, 0, 64, 256, 0, 256, FAKE, FAKE, 0, 256, None, None, 0, FAKE, 0, FAKE, 1 << 30, None]

    def call(**over):
        a = list(ok)
        for k, v in over.items():
            a[names.index(k)] = v
        return L.convrot_linear_ex(*a)

    assert call(dtype=2) == 2                      # unknown dtype
    assert call(mode=2) == 2                       # unknown scale mode
    assert call(act=7) == 2                        # unknown activation
    assert call(mode=1, w_scale=FAKE + 4) == 1     # per-channel scales need 16-byte alignment
    assert call(addend=FAKE + 8) == 1              # misaligned addend
    assert call(ldx=200) == 1                      # ldx < K
    assert call(ldx=260) == 1                      # ldx not a multiple of 8
    assert call(ldy=255) == 1                      # ldy < N
    assert call(ldy=260) == 1                      # ldy not a multiple of 8
    assert call(g=64) == 2
    assert call(Y=None) == 1
    assert call(ws_bytes=100) == 3
    # prepare_weight_ex(W, dtype, N, K, g, mode, Wq, w_scale, ws, ws_bytes, stream)
    assert L.convrot_prepare_weight_ex(FAKE, 3, 8, 256, 256, 0, FAKE, FAKE, FAKE, 256, None) == 2
    assert L.convrot_prepare_weight_ex(FAKE, 0, 8, 256, 256, 5, FAKE, FAKE, FAKE, 256, None) == 2
    assert L.convrot_prepare_weight_ex(FAKE, 1, 8, 256, 256, 1, FAKE, FAKE + 4, None, 0, None) == 1
    assert L.convrot_prepare_weight_ex(FAKE, 1, 8, 256, 256, 0, FAKE, FAKE, None, 0, None) == 3
    # quant_act_ex(X, dtype, M, K, ldx, g, Xq, x_scale, stream)
    assert L.convrot_quant_act_ex(FAKE, 9, 8, 256, 0, 256, FAKE, FAKE, None) == 2
    assert L.convrot_quant_act_ex(FAKE, 1, 8, 300, 0, 256, FAKE, FAKE, None) == 1
    assert L.convrot_quant_act_ex(FAKE, 1, 8, 256, 100, 256, FAKE, FAKE, None) == 1


def test_empty_batch_is_a_checked_no_op_on_host(L):
    """M = 0 (no tokens) returns OK and enqueues nothing; the other arguments are still checked.

    There is no GPU here, so any CUDA call the library made would fail and return
    CONVROT_ERR_CUDA (4): an OK with null data pointers and a null workspace shows
    that nothing was launched or copied.
    """
    # convrot_linear(X, M, K, g, Wq, w_scale, N, bias, Y, ws, ws_bytes, stream)
    assert L.convrot_linear(None, 0, 3072, 256, FAKE, FAKE, 9216, None, None, None, 0, None) == 0
    assert L.convrot_linear(None, 0, 3072, 64, FAKE, FAKE, 9216, None, None, None, 0, None) == 2     # g
    assert L.convrot_linear(None, 0, 3000, 256, FAKE, FAKE, 9216, None, None, None, 0, None) == 1    # K % g
    assert L.convrot_linear(None, 0, 3072, 256, FAKE, FAKE, 0, None, None, None, 0, None) == 1       # N = 0
    assert L.convrot_linear(None, 0, 3072, 256, FAKE, FAKE, 9212, None, None, None, 0, None) == 1    # N % 8
    assert L.convrot_linear(None, -1, 3072, 256, FAKE, FAKE, 9216, None, None, None, 0, None) == 1   # M < 0
    assert L.convrot_linear_one_launch(None, 0, 3072, 256, FAKE, FAKE, 9216, None, None, None, 0, None) == 0
    assert L.convrot_linear_one_launch(None, 0, 20608, 128, FAKE, FAKE, 256, None, None, None, 0, None) == 2
    assert L.convrot_linear_noalloc(None, 0, 3072, 256, FAKE, FAKE, 9216, None, None, None, None) == 0
    assert L.convrot_linear_noalloc(None, 0, 3000, 256, FAKE, FAKE, 9216, None, None, None, None) == 1
    assert L.convrot_linear_launch_count(0, 9216, 3072, 256) == 0
    # convrot_linear_ex(X, dtype, M, K, ldx, g, Wq, w_scale, mode, N, bias, addend, act, Y, ldy, ws, ws_bytes, s)
    assert L.convrot_linear_ex(None, 1, 0, 256, 0, 256, FAKE, FAKE, 1, 256, None, None, 1, None, 0, None, 0,
                               None) == 0
    assert L.convrot_linear_ex(None, 1, 0, 256, 260, 256, FAKE, FAKE, 1, 256, None, None, 1, None, 0, None, 0,
                               None) == 1                                                          # ldx % 8
    assert L.convrot_linear_ex(None, 2, 0, 256, 0, 256, FAKE, FAKE, 0, 256, None, None, 0, None, 0, None, 0,
                               None) == 2                                                          # dtype
    assert L.convrot_quant_act(None, 0, 256, 256, None, None, None) == 0
    assert L.convrot_quant_act(None, 0, 256, 512, None, None, None) == 2
    assert L.convrot_quant_act_ex(None, 1, 0, 256, 264, 256, None, None, None) == 0
    assert L.convrot_quant_act_ex(None, 1, 0, 256, 100, 256, None, None, None) == 1
    assert L.convrot_gemm_dequant(None, None, FAKE, FAKE, 0, 8, 256, None, None, None, 0, None) == 0
    assert L.convrot_gemm_dequant(None, None, FAKE, FAKE, 0, 8, 24, None, None, None, 0, None) == 1  # K % 16
    assert L.convrot_gemm_s32(None, FAKE, 0, 8, 256, None, None, 0, None) == 0
    # a weight still has at least one output channel
    assert L.convrot_prepare_weight(FAKE, 0, 256, 256, FAKE, FAKE, FAKE, 256, None) == 1
    assert L.convrot_prepare_weight_ex(FAKE, 0, 0, 256, 256, 1, FAKE, FAKE, None, 0, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from w8a8_rotated_int8_token_b200 import _lib

    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.load()


def test_ctypes_signatures_match_header_arity():
    from w8a8_rotated_int8_token_b200 import _lib

    with open(os.path.join(ROOT, "include", "convrot.h")) as f:
        src = f.read()
    for name, (_, args) in _lib.SIGNATURES.items():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", src)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(args), name
    assert ctypes.sizeof(ctypes.c_size_t) == 8
