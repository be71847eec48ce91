"""INT8 ConvRot linear layer for NVIDIA B200 (sm_100a).

Python binding of libconvrot (include/convrot.h). Each function has the name
of the C entry point it calls and only marshals arguments: torch tensors are
passed as device pointers, the current CUDA stream as the stream. Outputs and
workspaces that the caller does not pass are allocated with torch (the
library itself never allocates). Every computation runs in the library's
CUDA kernels; there is no CPU path.

    Wq, s_w = convrot_prepare_weight(W, g=256)         # once per layer
    Y = convrot_linear(X, Wq, s_w, g=256, bias=b)     # per call
"""

from __future__ import annotations

from . import _lib

__all__ = [
    "ConvRotError",
    "convrot_abi_version",
    "convrot_status_string",
    "convrot_prepare_weight",
    "convrot_quant_act",
    "convrot_linear_workspace_bytes",
    "convrot_linear",
    "convrot_linear_one_launch",
    "convrot_prepare_weight_ex",
    "convrot_quant_act_ex",
    "convrot_linear_ex",
    "DTYPE_BF16",
    "DTYPE_F16",
    "WSCALE_TENSOR",
    "WSCALE_CHANNEL",
    "ACT_NONE",
    "ACT_GELU_ERF",
    "convrot_gemm_dequant",
    "convrot_gemm_s32",
    "convrot_read_device_status",
    "convrot_test_wait_timeout",
    "convrot_probe_i8_peak",
    "convrot_attention_workspace_bytes",
    "convrot_attention_int8",
    "ConvRotLinear",
    "lib",
]

# convrot_dtype, convrot_wscale_mode, convrot_activation (include/convrot.h)
DTYPE_BF16, DTYPE_F16 = 0, 1
WSCALE_TENSOR, WSCALE_CHANNEL = 0, 1
ACT_NONE, ACT_GELU_ERF = 0, 1

STATUS_NAMES = {0: "CONVROT_OK", 1: "CONVROT_ERR_INVALID_ARG", 2: "CONVROT_ERR_UNSUPPORTED",
                3: "CONVROT_ERR_WORKSPACE", 4: "CONVROT_ERR_CUDA", 5: "CONVROT_ERR_DEVICE_TIMEOUT"}


class ConvRotError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({convrot_status_string(status)})")


def lib():
    """The loaded ctypes library (raises ImportError if it is not built)."""
    return _lib.load()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise ConvRotError(status, where)


def _stream_ptr(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _require(t, dtype, shape, name):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def convrot_abi_version() -> int:
    return int(lib().convrot_abi_version())


def convrot_status_string(status: int) -> str:
    return lib().convrot_status_string(int(status)).decode()


def convrot_prepare_weight(W, g: int = 256, Wq=None, w_scale=None, ws=None, stream=None):
    """Rotate and quantise a bf16 weight [N,K]: returns (Wq int8 [N,K], w_scale float32 [1])."""
    import torch

    _require(W, torch.bfloat16, None, "W")
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty((1,), dtype=torch.float32, device=W.device)
    L = lib()
    if ws is None:
        ws = torch.empty((L.convrot_prepare_weight_workspace_bytes(),), dtype=torch.uint8, device=W.device)
    _require(Wq, torch.int8, (N, K), "Wq")
    _require(w_scale, torch.float32, (1,), "w_scale")
    _check(L.convrot_prepare_weight(_ptr(W), N, K, g, _ptr(Wq), _ptr(w_scale), _ptr(ws), ws.numel(),
                                    _stream_ptr(stream)), "convrot_prepare_weight")
    return Wq, w_scale


def convrot_quant_act(X, g: int = 256, Xq=None, x_scale=None, stream=None):
    """Rotate + per-token quantise bf16 X [M,K]: returns (Xq int8 [M,K], x_scale float32 [M])."""
    import torch

    _require(X, torch.bfloat16, None, "X")
    M, K = X.shape
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if x_scale is None:
        x_scale = torch.empty((M,), dtype=torch.float32, device=X.device)
    _require(Xq, torch.int8, (M, K), "Xq")
    _require(x_scale, torch.float32, (M,), "x_scale")
    _check(lib().convrot_quant_act(_ptr(X), M, K, g, _ptr(Xq), _ptr(x_scale), _stream_ptr(stream)),
           "convrot_quant_act")
    return Xq, x_scale


def convrot_linear_workspace_bytes(M: int, N: int, K: int, g: int) -> int:
    return int(lib().convrot_linear_workspace_bytes(M, N, K, g))


def convrot_linear(X, Wq, w_scale, g: int = 256, bias=None, Y=None, ws=None, stream=None):
    """Y [M,N] bf16 = ConvRot linear of bf16 X [M,K] with the prepared weight (Wq, w_scale)."""
    import torch

    _require(X, torch.bfloat16, None, "X")
    M, K = X.shape
    _require(Wq, torch.int8, None, "Wq")
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError("Wq must be [N, K] with the K of X")
    _require(w_scale, torch.float32, (1,), "w_scale")
    if bias is not None:
        _require(bias, torch.bfloat16, (N,), "bias")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    need = convrot_linear_workspace_bytes(M, N, K, g)
    if ws is None:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=X.device)
    _check(lib().convrot_linear(_ptr(X), M, K, g, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), _ptr(Y), _ptr(ws),
                                ws.numel(), _stream_ptr(stream)), "convrot_linear")
    return Y


def convrot_linear_one_launch(X, Wq, w_scale, g: int = 256, bias=None, Y=None, ws=None, stream=None):
    """convrot_linear as one kernel launch (rotate+quantise workers inside the GEMM kernel; K <= 20480)."""
    import torch

    _require(X, torch.bfloat16, None, "X")
    M, K = X.shape
    _require(Wq, torch.int8, None, "Wq")
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError("Wq must be [N, K] with the K of X")
    _require(w_scale, torch.float32, (1,), "w_scale")
    if bias is not None:
        _require(bias, torch.bfloat16, (N,), "bias")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    need = convrot_linear_workspace_bytes(M, N, K, g)
    if ws is None:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=X.device)
    _check(lib().convrot_linear_one_launch(_ptr(X), M, K, g, _ptr(Wq), _ptr(w_scale), N, _ptr(bias), _ptr(Y),
                                           _ptr(ws), ws.numel(), _stream_ptr(stream)), "convrot_linear_one_launch")
    return Y


def _dtype_code(t, name):
    import torch

    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float16:
        return DTYPE_F16
    raise TypeError(f"{name}: expected bfloat16 or float16, got {t.dtype}")


def convrot_prepare_weight_ex(W, g: int = 256, wscale_mode: int = WSCALE_TENSOR, Wq=None, w_scale=None, ws=None,
                              stream=None):
    """Rotate and quantise a bf16 or fp16 weight [N,K]: returns (Wq int8 [N,K], w_scale float32 [1] or [N])."""
    import torch

    dtype = _dtype_code(W, "W")
    _require(W, W.dtype, None, "W")
    N, K = W.shape
    ns = N if wscale_mode == WSCALE_CHANNEL else 1
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if w_scale is None:
        w_scale = torch.empty((ns,), dtype=torch.float32, device=W.device)
    L = lib()
    if ws is None and wscale_mode != WSCALE_CHANNEL:
        ws = torch.empty((L.convrot_prepare_weight_workspace_bytes(),), dtype=torch.uint8, device=W.device)
    _require(Wq, torch.int8, (N, K), "Wq")
    _require(w_scale, torch.float32, (ns,), "w_scale")
    _check(L.convrot_prepare_weight_ex(_ptr(W), dtype, N, K, g, int(wscale_mode), _ptr(Wq), _ptr(w_scale), _ptr(ws),
                                       0 if ws is None else ws.numel(), _stream_ptr(stream)),
           "convrot_prepare_weight_ex")
    return Wq, w_scale


def _rows_view(t, name):
    """(rows, cols, row stride in elements) of a 2-D tensor whose rows may be strided."""
    import torch

    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D CUDA tensor with contiguous rows")
    return t.shape[0], t.shape[1], t.stride(0)


def convrot_quant_act_ex(X, g: int = 256, Xq=None, x_scale=None, stream=None):
    """convrot_quant_act for a bf16 or fp16 X [M,K] whose rows may be strided."""
    import torch

    dtype = _dtype_code(X, "X")
    M, K, ldx = _rows_view(X, "X")
    if Xq is None:
        Xq = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if x_scale is None:
        x_scale = torch.empty((M,), dtype=torch.float32, device=X.device)
    _require(Xq, torch.int8, (M, K), "Xq")
    _require(x_scale, torch.float32, (M,), "x_scale")
    _check(lib().convrot_quant_act_ex(_ptr(X), dtype, M, K, ldx, g, _ptr(Xq), _ptr(x_scale), _stream_ptr(stream)),
           "convrot_quant_act_ex")
    return Xq, x_scale


def convrot_linear_ex(X, Wq, w_scale, g: int = 256, bias=None, activation: int = ACT_NONE, Y=None, ws=None,
                      stream=None, addend=None):
    """ConvRot linear in the dtype of X (bf16 or fp16; bias, addend and Y the same), with a
    tensor (w_scale [1]) or per-output-channel (w_scale [N]) weight scale, an optional
    addend [M,N] (a term computed beside the int8 layer, e.g. a LoRA's output) and an
    optional exact-erf GELU. X, Y and addend may have strided rows (Y and addend share
    one row stride)."""
    import torch

    dtype = _dtype_code(X, "X")
    M, K, ldx = _rows_view(X, "X")
    _require(Wq, torch.int8, None, "Wq")
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError("Wq must be [N, K] with the K of X")
    if w_scale.numel() == N and N != 1:
        mode = WSCALE_CHANNEL
    elif w_scale.numel() == 1:
        mode = WSCALE_TENSOR
    else:
        raise ValueError("w_scale must hold 1 or N floats")
    _require(w_scale, torch.float32, (w_scale.numel(),), "w_scale")
    if bias is not None:
        _require(bias, X.dtype, (N,), "bias")
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    if Y.dtype != X.dtype or tuple(Y.shape) != (M, N):
        raise ValueError(f"Y must be [{M}, {N}] {X.dtype}")
    _, _, ldy = _rows_view(Y, "Y")
    if addend is not None:
        if addend.dtype != X.dtype or tuple(addend.shape) != (M, N) or _rows_view(addend, "addend")[2] != ldy:
            raise ValueError("addend must be [M, N] in the dtype of X, with the row stride of Y")
    need = convrot_linear_workspace_bytes(M, N, K, g)
    if ws is None:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=X.device)
    _check(lib().convrot_linear_ex(_ptr(X), dtype, M, K, ldx, g, _ptr(Wq), _ptr(w_scale), mode, N, _ptr(bias),
                                   _ptr(addend), int(activation), _ptr(Y), ldy, _ptr(ws), ws.numel(),
                                   _stream_ptr(stream)), "convrot_linear_ex")
    return Y


def convrot_gemm_dequant(Xq, x_scale, Wq, w_scale, bias=None, Y=None, ws=None, stream=None):
    """GEMM + epilogue on already-quantised codes: Y [M,N] bf16."""
    import torch

    _require(Xq, torch.int8, None, "Xq")
    M, K = Xq.shape
    _require(Wq, torch.int8, None, "Wq")
    N = Wq.shape[0]
    _require(x_scale, torch.float32, (M,), "x_scale")
    _require(w_scale, torch.float32, (1,), "w_scale")
    if bias is not None:
        _require(bias, torch.bfloat16, (N,), "bias")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _require(Y, torch.bfloat16, (M, N), "Y")
    L = lib()
    if ws is None:
        ws = torch.empty((L.convrot_gemm_workspace_bytes(),), dtype=torch.uint8, device=Xq.device)
    _check(L.convrot_gemm_dequant(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, _ptr(bias), _ptr(Y),
                                  _ptr(ws), ws.numel(), _stream_ptr(stream)), "convrot_gemm_dequant")
    return Y


def convrot_gemm_s32(Xq, Wq, acc=None, ws=None, stream=None):
    """Raw int32 accumulators acc [M,N] = Xq Wq^T from the tcgen05 GEMM."""
    import torch

    _require(Xq, torch.int8, None, "Xq")
    M, K = Xq.shape
    _require(Wq, torch.int8, None, "Wq")
    N = Wq.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=Xq.device)
    _require(acc, torch.int32, (M, N), "acc")
    L = lib()
    if ws is None:
        ws = torch.empty((L.convrot_gemm_workspace_bytes(),), dtype=torch.uint8, device=Xq.device)
    _check(L.convrot_gemm_s32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), _ptr(ws), ws.numel(), _stream_ptr(stream)),
           "convrot_gemm_s32")
    return acc


def convrot_read_device_status(ws, stream=None) -> int:
    """Status word of a workspace (synchronises the stream): 0 or CONVROT_ERR_DEVICE_TIMEOUT (5)."""
    return int(lib().convrot_read_device_status(_ptr(ws), _stream_ptr(stream)))


def convrot_test_wait_timeout(ws, timeout_ns: int, stream=None) -> None:
    _check(lib().convrot_test_wait_timeout(_ptr(ws), ws.numel(), int(timeout_ns), _stream_ptr(stream)),
           "convrot_test_wait_timeout")


def convrot_probe_i8_peak(iters: int, operands=None, ws=None, stream=None) -> int:
    """Enqueue the int8 tensor-pipe peak probe (one CTA pair per two SMs, `iters` x 4
    tcgen05.mma.cta_group::2.kind::i8 of 256x256x32 each, no global traffic in the loop);
    returns the number of CTAs launched. `operands`: None (zero operands) or a contiguous
    device tensor whose bytes fill the CTAs' operand tiles. The caller times it with
    events on `stream`."""
    import torch

    L = lib()
    if ws is None:
        ws = torch.empty((256,), dtype=torch.uint8, device=torch.cuda.current_device())
    op_ptr, op_bytes = None, 0
    if operands is not None:
        if not operands.is_contiguous():
            raise ValueError("operands must be contiguous")
        op_ptr, op_bytes = _ptr(operands), operands.numel() * operands.element_size()
    _check(L.convrot_probe_i8_peak(int(iters), op_ptr, op_bytes, _ptr(ws), ws.numel(), _stream_ptr(stream)),
           "convrot_probe_i8_peak")
    return int(L.convrot_probe_i8_peak_ctas())


def convrot_attention_workspace_bytes(BH: int, Sq: int, Skv: int, D: int = 128) -> int:
    return int(lib().convrot_attention_workspace_bytes(BH, Sq, Skv, D))


def convrot_attention_int8(Q, K, V, softmax_scale=None, O=None, ws=None, stream=None):
    """INT8 attention of bf16 Q [..., Sq, 128] with K, V [..., Skv, 128] (same leading
    dims, flattened to batch*heads): O [..., Sq, 128] bf16 (see include/convrot.h)."""
    import math

    import torch

    for t, name in ((Q, "Q"), (K, "K"), (V, "V")):
        _require(t, torch.bfloat16, None, name)
        if t.dim() < 2 or t.shape[-1] != 128:
            raise ValueError(f"{name} must be [..., S, 128]")
    lead = tuple(Q.shape[:-2])
    if tuple(K.shape[:-2]) != lead or tuple(V.shape) != tuple(K.shape):
        raise ValueError("Q, K and V must share their leading dimensions, and K and V their shape")
    Sq, Skv, D = Q.shape[-2], K.shape[-2], Q.shape[-1]
    BH = int(math.prod(lead)) if lead else 1
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16, device=Q.device)
    _require(O, torch.bfloat16, tuple(Q.shape), "O")
    need = convrot_attention_workspace_bytes(BH, Sq, Skv, D)
    if ws is None:
        ws = torch.empty((max(need, 256),), dtype=torch.uint8, device=Q.device)
    _check(lib().convrot_attention_int8(_ptr(Q), _ptr(K), _ptr(V), BH, Sq, Skv, D, float(softmax_scale), _ptr(O),
                                        _ptr(ws), ws.numel(), _stream_ptr(stream)), "convrot_attention_int8")
    return O


class ConvRotLinear:
    """A ConvRot linear layer: prepared int8 weight + optional bias, reusable workspace.

    ``layer = ConvRotLinear(W, bias, g=256)`` rotates and quantises W once;
    ``layer(X)`` runs convrot_linear on the current stream. With a float16 W,
    ``wscale_mode=WSCALE_CHANNEL`` or ``activation=ACT_GELU_ERF`` the layer
    runs convrot_linear_ex instead (X, bias and Y then share W's dtype), and
    ``layer(X, addend=Z)`` adds Z [M,N] before the activation.
    """

    def __init__(self, W, bias=None, g: int = 256, wscale_mode: int = WSCALE_TENSOR, activation: int = ACT_NONE):
        import torch

        self.g = g
        self.N, self.K = W.shape
        self.activation = int(activation)
        self.general = W.dtype != torch.bfloat16 or wscale_mode != WSCALE_TENSOR or self.activation != ACT_NONE
        if self.general:
            self.Wq, self.w_scale = convrot_prepare_weight_ex(W, g, wscale_mode)
        else:
            self.Wq, self.w_scale = convrot_prepare_weight(W, g)
        self.bias = bias
        self._ws = None

    def workspace(self, M: int):
        import torch

        need = convrot_linear_workspace_bytes(M, self.N, self.K, self.g)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=self.Wq.device)
        return self._ws

    def __call__(self, X, Y=None, stream=None, addend=None):
        ws = self.workspace(X.shape[0])
        if self.general or addend is not None:
            return convrot_linear_ex(X, self.Wq, self.w_scale, self.g, self.bias, self.activation, Y, ws, stream,
                                     addend)
        return convrot_linear(X, self.Wq, self.w_scale, self.g, self.bias, Y, ws, stream)
