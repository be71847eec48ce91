"""Seeded synthetic inputs shaped like diffusion-transformer and text-encoder layers.

The workloads stand in for the layers that the int8 compute measurements run
(FLUX.1-dev / Z-Image / Krea-2 denoisers at 1024^2 and 2048^2, and a ConvRot
int8 text encoder; InvokeAI "int8 Compute" page, opening section and its
timing table). The pages give no layer shapes, so the token counts and widths
below are the standard DiT shapes for those resolutions (4096 image + 512 text
tokens at 1024^2, 16384 + 512 at 2048^2, width 3072, fused QKV 9216, MLP 12288)
and a text encoder of width 4096.

Recipe (identical for every config; only the numbers in the table change):
  1. ``rng = numpy.random.default_rng(seed)`` (PCG64).
  2. X: ``rng.standard_normal((M, K), float32)``, or Student-t(nu=4) for the
     heavy-tailed 2048^2 layer, drawn as float64 and cast to float32.
  3. Outlier channels: ``rng.choice(K, floor(frac * K), replace=False)``; the
     whole column is multiplied by the outlier factor.
  4. W: ``rng.standard_normal((N, K), float32) * w_std``.
  5. bias (only where the config has one): ``rng.standard_normal(N, float32) * 0.01``.
  6. Every tensor is rounded to bf16 (round-to-nearest-even) and kept as its
     uint16 bit pattern; both sides of a comparison read those same bits.

The DiT MLP down-projection takes the GELU of the up-projection's output as its
input; ``gelu_bf16_bits`` turns a given up-projection output into that input.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    N: int
    g: int
    seed: int
    x_dist: str          # "normal" | "student_t4" | "gelu_of_up"
    outlier_frac: float  # fraction of K channels that are outliers
    outlier_mult: float
    w_std: float
    bias: bool

    def gemm_ops(self) -> int:
        return 2 * self.M * self.N * self.K


# The five layer shapes. The text-encoder layer is run at four token counts.
CONFIGS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 64, 256, 256, 256, 0, "normal", 4 / 256, 30.0, 0.02, False),
        Workload("dit_qkv_1024", 4608, 3072, 9216, 256, 1, "normal", 0.01, 50.0, 0.02, True),
        Workload("dit_mlp_up_1024", 4608, 3072, 12288, 256, 2, "normal", 0.01, 50.0, 0.02, False),
        Workload("dit_mlp_down_1024", 4608, 12288, 3072, 256, 5, "gelu_of_up", 0.0, 1.0, 0.02, False),
        Workload("dit_mlp_2048", 16896, 3072, 12288, 256, 3, "student_t4", 0.01, 50.0, 0.02, False),
        Workload("textenc_m1", 1, 4096, 12288, 128, 4, "normal", 0.005, 100.0, 0.015, False),
        Workload("textenc_m16", 16, 4096, 12288, 128, 4, "normal", 0.005, 100.0, 0.015, False),
        Workload("textenc_m128", 128, 4096, 12288, 128, 4, "normal", 0.005, 100.0, 0.015, False),
        Workload("textenc_m512", 512, 4096, 12288, 128, 4, "normal", 0.005, 100.0, 0.015, False),
    ]
}

# The text-encoder configs share one weight and take the first M rows of one
# 512-token activation draw, so that M=1/16/128 are prefixes of M=512.
_TEXTENC_ROWS = 512


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen uint16 bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def gelu_bf16_bits(y: np.ndarray) -> np.ndarray:
    """Input of the DiT MLP down-projection: bf16(GELU(bf16(y))), exact-erf GELU.

    ``y`` is the up-projection output (any float dtype). It is first rounded
    to bf16 (what the layer would store), then GELU is taken in float64 and
    the result rounded to bf16 via float32.
    """
    from scipy.special import erf  # only this helper needs scipy

    yb = bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(y, dtype=np.float32))).astype(np.float64)
    gl = 0.5 * yb * (1.0 + erf(yb / math.sqrt(2.0)))
    return f32_to_bf16_bits(gl.astype(np.float32))


def _draw_x(rng: np.random.Generator, w: Workload, rows: int) -> np.ndarray:
    if w.x_dist == "normal":
        x = rng.standard_normal((rows, w.K), dtype=np.float32)
    elif w.x_dist == "student_t4":
        x = rng.standard_t(4.0, size=(rows, w.K)).astype(np.float32)
    else:
        raise ValueError(f"{w.name}: X is derived from another layer's output")
    n_out = int(math.floor(w.outlier_frac * w.K))
    if n_out:
        ch = rng.choice(w.K, n_out, replace=False)
        x[:, ch] *= np.float32(w.outlier_mult)
    return x


def make_workload(name: str, x_up_output: np.ndarray | None = None,
                  rows: int | None = None) -> dict:
    """Draw one config's tensors as bf16 bits.

    Returns a dict with ``x`` [M,K], ``w`` [N,K], ``bias`` [N] or None (all
    uint16 bf16 bits) and the ``workload`` record. ``rows`` draws only the
    first ``rows`` tokens of X where the draw allows it (the weight and bias
    are unchanged); for the down-projection the caller passes the
    up-projection output in ``x_up_output``.
    """
    w = CONFIGS[name]
    rng = np.random.default_rng(w.seed)
    if w.x_dist == "gelu_of_up":
        if x_up_output is None:
            raise ValueError("dit_mlp_down_1024 needs the up-projection output")
        xb = gelu_bf16_bits(x_up_output)
        if xb.shape[1] != w.K:
            raise ValueError("up-projection output width does not match K")
        # the down-projection's own draws: its weight only (its own seed, so
        # that it is not a rescaled copy of the up-projection's activations)
        wt = rng.standard_normal((w.N, w.K), dtype=np.float32) * np.float32(w.w_std)
        bias = None
    else:
        m_draw = _TEXTENC_ROWS if name.startswith("textenc") else w.M
        x = _draw_x(rng, w, m_draw)
        wt = rng.standard_normal((w.N, w.K), dtype=np.float32) * np.float32(w.w_std)
        bias = (rng.standard_normal(w.N, dtype=np.float32) * np.float32(0.01)) if w.bias else None
        x = x[: w.M]
        xb = f32_to_bf16_bits(x)
    if rows is not None:
        xb = xb[:rows]
    return {
        "workload": w,
        "x": np.ascontiguousarray(xb),
        "w": f32_to_bf16_bits(wt),
        "bias": None if bias is None else f32_to_bf16_bits(bias),
    }
