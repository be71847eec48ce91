"""CPU oracle of the INT8 ConvRot linear layer (plain NumPy, float64).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The library under
``w8a8_rotated_int8_token_b200/`` never calls it and has no CPU path of its own.
This module shares no code with the CUDA path and imports nothing from it.

What one call computes (the pages' description, restated):
  * The weight of a ConvRot layer is stored as int8 with one scale for the
    whole tensor ("int8_tensorwise"; InvokeAI "int8 Compute" page, opening
    section).
  * Each call rotates its input, quantises it to int8 with one scale per token,
    and multiplies int8 by int8 (same page, second paragraph).
  * The rotation acts on groups of input channels, 256 wide in every published
    build (same page, "What stays on the default path"); it is a group-wise
    rotation applied block by block along the channel axis, which spreads an
    outlier channel over its group ("Explanation of INT8 ConvRot", section
    "What is INT8 ConvRot?").
  * Rounding is round-to-nearest ("RTN" in the format tables of that article,
    section "Representative Model Formats and INT8 ConvRot").

Readings where the pages are silent (each listed in the design notes):
  * The rotation is the orthonormal Sylvester Walsh-Hadamard matrix H_g/sqrt(g),
    H[i, j] = (-1)^popcount(i & j), applied to every length-g block of K, with
    no sign flips or permutation. The same R rotates the weight rows, so
    X R (W R)^T = X W^T.
  * Quantisation is symmetric with codes in [-127, 127]; ties round to even;
    an all-zero token gets scale 0 and codes 0.
  * The weight scale is one float32 for the whole tensor; the activation scale
    is one float32 per token (row).
  * Dequantisation: y = acc * (s_x[m] * s_w) + bias[n].
  * Variants: an FP16 compute dtype (X, bias and Y in fp16), one weight scale
    per output channel, and an exact-erf GELU applied to y (the MLP
    up-projection with its activation fused).

Every step is written from its definition: the rotation is an explicit matrix
product (no butterflies), the GEMM is a float64 matrix product of integer
codes (exact, since every partial sum is an integer below 2^53), and nothing
is blocked, fused or reordered.
"""

from __future__ import annotations

import numpy as np

QMAX = 127


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 values given as uint16 bit patterns, widened exactly to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE fp16 values given as uint16 bit patterns, widened exactly to float64.

    The layer's compute dtype may be FP16 as well as BF16 (InvokeAI "int8
    Compute" page, "What stays on the default path": the kernels run in BF16
    and FP16 only).
    """
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def hadamard(g: int) -> np.ndarray:
    """Sylvester-ordered Hadamard matrix H_g with entries (-1)^popcount(i & j).

    Reading of the "group-based rotation" of the ConvRot article (section
    "What is INT8 ConvRot?"): the orthogonal matrix of each group is H_g/sqrt(g).
    """
    if g < 1 or g & (g - 1):
        raise ValueError("group size must be a power of two")
    i = np.arange(g, dtype=np.int64)
    anded = i[:, None] & i[None, :]
    parity = np.zeros_like(anded)
    v = anded.copy()
    while np.any(v):
        parity ^= v & 1
        v >>= 1
    return np.where(parity == 1, -1.0, 1.0)


def rotation_matrix(K: int, g: int) -> np.ndarray:
    """The full K x K rotation R = blockdiag(H_g/sqrt(g), ..., H_g/sqrt(g)).

    Only for small K (it is dense); ``rotate`` applies the same matrix block
    by block.
    """
    if K % g:
        raise ValueError("K must be a multiple of the group size")
    return np.kron(np.eye(K // g), hadamard(g) / np.sqrt(g))


def rotate(x: np.ndarray, g: int) -> np.ndarray:
    """x R for row vectors x (last axis K): each length-g block times H_g/sqrt(g).

    The group rotation of the ConvRot article ("What is INT8 ConvRot?"), the
    same g x g matrix slid over K in non-overlapping blocks. Float64.
    """
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if K % g:
        raise ValueError("K must be a multiple of the group size")
    blocks = x.reshape(x.shape[:-1] + (K // g, g))
    return (blocks @ (hadamard(g) / np.sqrt(g))).reshape(x.shape)


def quantize_per_token(xr: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-token symmetric int8 quantisation of already-rotated rows.

    s[m] = float32(max_k |xr[m, k]| / 127); codes = clip(rint(xr / s), -127, 127)
    with the division in float64 by the float32 scale, rint rounding ties to
    even; a row whose absmax is 0 gets s = 0 and all-zero codes. (InvokeAI
    "int8 Compute", second paragraph: one scale per token.)
    """
    xr = np.asarray(xr, dtype=np.float64)
    amax = np.max(np.abs(xr), axis=-1)
    s = (amax / QMAX).astype(np.float32)
    s64 = s.astype(np.float64)
    safe = np.where(s64 > 0, s64, 1.0)
    q = np.rint(xr / safe[..., None])
    q = np.where(s64[..., None] > 0, q, 0.0)
    q = np.clip(q, -QMAX, QMAX)
    return q.astype(np.int8), s


def quantize_tensorwise(wr: np.ndarray) -> tuple[np.ndarray, np.float32]:
    """Tensorwise symmetric int8 quantisation of the rotated weight.

    s_w = float32(max |wr| / 127); codes = clip(rint(wr / s_w), -127, 127)
    ("int8_tensorwise" on the InvokeAI "int8 Compute" page, opening section).
    """
    wr = np.asarray(wr, dtype=np.float64)
    s = np.float32(np.max(np.abs(wr)) / QMAX)
    if s == 0:
        return np.zeros(wr.shape, np.int8), s
    q = np.clip(np.rint(wr / np.float64(s)), -QMAX, QMAX)
    return q.astype(np.int8), s


def prepare_weight(w: np.ndarray, g: int) -> tuple[np.ndarray, np.float32]:
    """W [N,K] (float values) -> (Wq int8 [N,K], s_w float32): rotate rows, then quantise."""
    return quantize_tensorwise(rotate(w, g))


def prepare_weight_per_channel(w: np.ndarray, g: int) -> tuple[np.ndarray, np.ndarray]:
    """W [N,K] -> (Wq int8 [N,K], s_w float32 [N]): rotate rows, one scale per output channel.

    The "Row-wise" scaling of INT8 ConvRot in the format table of the ConvRot
    article (section "Representative Model Formats and INT8 ConvRot"), read as
    one scale per weight row (output channel): the same symmetric rule as the
    per-token activation scale, applied to the rows of W R.
    """
    return quantize_per_token(rotate(w, g))


def quant_act(x: np.ndarray, g: int) -> tuple[np.ndarray, np.ndarray]:
    """X [M,K] (float values) -> (Xq int8 [M,K], s_x float32 [M]): rotate tokens, then quantise."""
    return quantize_per_token(rotate(x, g))


def gemm_s32(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k xq[m, k] * wq[n, k] as int32 (int8 x int8, int32 accumulate).

    The float64 product of integer codes is exact: |every partial sum| <=
    K * 127^2 < 2^53. Raises if a result does not fit int32.
    """
    acc = np.asarray(xq, np.float64) @ np.asarray(wq, np.float64).T
    if acc.size and np.max(np.abs(acc)) >= 2.0**31:
        raise OverflowError("accumulator exceeds int32")
    return acc.astype(np.int32)


def dequant(acc: np.ndarray, s_x: np.ndarray, s_w: float, bias: np.ndarray | None = None) -> np.ndarray:
    """y[m, n] = acc[m, n] * (s_x[m] * s_w) + bias[n], in float64."""
    y = np.asarray(acc, np.float64) * (np.asarray(s_x, np.float64)[:, None] * np.float64(s_w))
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y


def dequant_per_channel(acc: np.ndarray, s_x: np.ndarray, s_w: np.ndarray,
                        bias: np.ndarray | None = None) -> np.ndarray:
    """y[m, n] = acc[m, n] * (s_x[m] * s_w[n]) + bias[n], in float64 (per-output-channel weight scale)."""
    y = np.asarray(acc, np.float64) * (np.asarray(s_x, np.float64)[:, None] * np.asarray(s_w, np.float64)[None, :])
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y


def gelu_erf(y: np.ndarray) -> np.ndarray:
    """GELU with the exact Gaussian CDF: y * Phi(y) = 0.5 * y * (1 + erf(y / sqrt(2))), float64.

    The activation between the two MLP projections of the diffusion
    transformers the pages measure; applied to the up projection's output
    when it is fused into that layer.
    """
    from scipy.special import erf

    y = np.asarray(y, np.float64)
    return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))


def linear_ex(x: np.ndarray, wq: np.ndarray, s_w, g: int, bias: np.ndarray | None = None,
              addend: np.ndarray | None = None, gelu: bool = False) -> np.ndarray:
    """The layer with its variants, float64: rotate + per-token quantise X, int8 GEMM,
    dequantise with a tensor (scalar s_w) or per-output-channel (s_w [N]) weight
    scale, add the bias, add `addend` [M,N] (a term computed beside the int8
    layer, as a LoRA is: InvokeAI "int8 Compute", after the list in "What stays
    on the default path": applied beside the int8 layer in the compute
    precision, never quantised), then GELU if asked.
    """
    xq, s_x = quant_act(x, g)
    acc = gemm_s32(xq, wq)
    s_w = np.asarray(s_w)
    y = dequant_per_channel(acc, s_x, s_w, bias) if s_w.ndim == 1 and s_w.size > 1 else dequant(acc, s_x, s_w, bias)
    if addend is not None:
        y = y + np.asarray(addend, np.float64)
    return gelu_erf(y) if gelu else y


def linear(x: np.ndarray, wq: np.ndarray, s_w: float, g: int,
           bias: np.ndarray | None = None) -> np.ndarray:
    """One ConvRot linear call: rotate + per-token quantise X, int8 GEMM, dequantise."""
    xq, s_x = quant_act(x, g)
    return dequant(gemm_s32(xq, wq), s_x, s_w, bias)


def to_bf16_rne(y: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); return uint16 bits.

    Used to show a result in the layer's output type. The value passes
    through float32 first, so the double rounding can only differ from a
    direct float64 -> bf16 rounding within 2^-24 relative of a bf16 tie;
    every comparison uses a tolerance far above that.
    """
    u = np.asarray(y, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def to_f16_rne(y: np.ndarray) -> np.ndarray:
    """Round float64 values to IEEE fp16 (nearest, ties to even); return uint16 bits.

    NumPy's float64 -> float16 cast rounds to nearest even directly.
    """
    with np.errstate(over="ignore"):  # values past the fp16 range round to infinity
        return np.asarray(y, np.float64).astype(np.float16).view(np.uint16)


def nrmse(y: np.ndarray, ref: np.ndarray) -> float:
    """||y - ref||_2 / ||ref||_2 over all elements, float64."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(y - ref)
    return float(num / den) if den > 0 else float(num)
