"""CPU oracle of INT8 attention (plain NumPy, float64).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module. The library never calls it
and has no CPU path of its own. It shares no code with the CUDA path.

What the pages give. The Hugging Face discussion "INT8 ConvRot on 2xT4"
(section "Attention kernel alone") times an INT8 attention call on 4096 image
tokens plus a 128-token prefix, 32 heads, head dimension 128, and reports its
NRMSE against FP32 attention; its section "Two things worth flagging" says the
error grows with the sequence length when the attention logits are large
(a logit scale of 4) and tracks the dynamic range of Q. The InvokeAI "int8
Compute" page (after its timing table) notes that attention is the part the
int8 linear layers leave in 16-bit. None of the pages gives the quantisation
scheme of the attention kernel.

Reading (the plainest one the rest supports; listed in the design notes):
  * Q and K are treated as the linear layer treats its activations: every
    token's head vector (length D = 128) is rotated by the normalised
    Walsh-Hadamard matrix H_D/sqrt(D) and quantised to int8 with one
    symmetric scale per token, absmax/127, ties to even. The same rotation on
    both sides leaves Q K^T unchanged.
  * S[i, j] = (q_i . k_j) * s_q[i] * s_k[j] * softmax_scale, with the integer
    dot product exact.
  * P = softmax over the keys of each query row; O = P V with V as given.
Every step is written from its definition with library matrix products; the
softmax subtracts the row maximum (an identity of the softmax) before exp.
"""

from __future__ import annotations

import numpy as np

from .convrot_oracle import quantize_per_token, rotate


def quantize_heads(x: np.ndarray, g: int) -> tuple[np.ndarray, np.ndarray]:
    """x [..., S, D] float values -> (codes int8 [..., S, D], scales float32 [..., S]):
    rotate each token's head vector in groups of g along D, then one scale per token."""
    x = np.asarray(x, np.float64)
    return quantize_per_token(rotate(x, g))


def softmax(s: np.ndarray) -> np.ndarray:
    """Row softmax over the last axis, float64 (the row maximum subtracted first)."""
    s = np.asarray(s, np.float64)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_logits(qc: np.ndarray, sq: np.ndarray, kc: np.ndarray, sk: np.ndarray,
                     softmax_scale: float) -> np.ndarray:
    """S = (qc kc^T) * s_q[:, None] * s_k[None, :] * softmax_scale over the last two axes.

    The integer product of the codes is exact in float64 (|partial sums| <= D * 127^2).
    """
    acc = np.asarray(qc, np.float64) @ np.swapaxes(np.asarray(kc, np.float64), -1, -2)
    return acc * (np.asarray(sq, np.float64)[..., :, None] * np.asarray(sk, np.float64)[..., None, :]) \
        * np.float64(softmax_scale)


def attention_int8(q: np.ndarray, k: np.ndarray, v: np.ndarray, softmax_scale: float | None = None,
                   g: int | None = None, return_parts: bool = False):
    """INT8 attention of q [..., Sq, D], k [..., Skv, D], v [..., Skv, D] (float values), float64.

    Returns O [..., Sq, D]; with ``return_parts`` also a dict with the codes,
    scales, logits and probabilities.
    """
    q = np.asarray(q, np.float64)
    D = q.shape[-1]
    g = D if g is None else g
    scale = (1.0 / np.sqrt(D)) if softmax_scale is None else float(softmax_scale)
    qc, sq = quantize_heads(q, g)
    kc, sk = quantize_heads(k, g)
    s = attention_logits(qc, sq, kc, sk, scale)
    p = softmax(s)
    o = p @ np.asarray(v, np.float64)
    if return_parts:
        return o, {"qc": qc, "sq": sq, "kc": kc, "sk": sk, "s": s, "p": p}
    return o


def attention_exact(q: np.ndarray, k: np.ndarray, v: np.ndarray, softmax_scale: float | None = None) -> np.ndarray:
    """Attention without quantisation (the FP32 reference of the pages' NRMSE, here in float64)."""
    q = np.asarray(q, np.float64)
    scale = (1.0 / np.sqrt(q.shape[-1])) if softmax_scale is None else float(softmax_scale)
    s = (q @ np.swapaxes(np.asarray(k, np.float64), -1, -2)) * scale
    return softmax(s) @ np.asarray(v, np.float64)
