"""Comparison helpers shared by the GPU parity tests (CUDA path vs the CPU oracle).

Tolerances (stated once, used everywhere):
  * int32 accumulators: bit-exact when both sides get the same int8 codes.
  * int8 codes: |delta| <= 1, on at most 1e-4 of the elements, and only where
    the oracle's float64 quotient lies within CODE_TIE_WINDOW of a rounding
    boundary (k + 0.5): the kernel rotates in float32 with a different
    summation order, so only near-ties may round the other way.
  * token / tensor scales: relative difference <= 1e-6.
  * bf16 output: NRMSE <= 2e-3 against the oracle's float64 result, and
    every element within the rounding bound of the oracle's arithmetic applied
    to the kernel's own codes and scales (``check_output_elementwise``): the
    one output rounding (half an ulp of bf16 or fp16) plus the float32
    dequantisation roundings, so that a single wrong element fails.
"""

from __future__ import annotations

import numpy as np

CODE_MISMATCH_FRAC = 1e-4
CODE_TIE_WINDOW = 1e-3
SCALE_RTOL = 1e-6
NRMSE_TOL = 2e-3


def to_torch_bf16(bits: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch

    u16 = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_codes(q_gpu: np.ndarray, s_gpu: np.ndarray, x_rot: np.ndarray, q_ref: np.ndarray, s_ref: np.ndarray,
                per_token: bool = True) -> dict:
    """Compare codes/scales of the kernel with the oracle's; return statistics.

    ``x_rot`` is the oracle's float64 rotated input, used to check that every
    differing code sits at a near-tie of the oracle's quotient.
    """
    s_gpu = np.asarray(s_gpu, np.float64)
    s_ref = np.asarray(s_ref, np.float64)
    denom = np.where(s_ref != 0, np.abs(s_ref), 1.0)
    rel = np.abs(s_gpu - s_ref) / denom
    assert np.all((s_ref == 0) == (s_gpu == 0)), "zero scales differ"
    assert rel.max(initial=0.0) <= SCALE_RTOL, f"scale rel diff {rel.max()}"
    d = q_gpu.astype(np.int32) - q_ref.astype(np.int32)
    assert np.abs(d).max(initial=0) <= 1, f"code differs by {np.abs(d).max()}"
    bad = np.nonzero(d)
    frac = len(bad[0]) / max(1, d.size)
    assert frac <= CODE_MISMATCH_FRAC, f"code mismatch fraction {frac}"
    if len(bad[0]):
        s_b = s_ref[bad[0]] if per_token else np.full(len(bad[0]), float(s_ref.reshape(-1)[0]))
        quot = x_rot[bad] / s_b
        tie_dist = np.abs(np.abs(quot - np.floor(quot)) - 0.5)
        assert tie_dist.max() <= CODE_TIE_WINDOW, f"a differing code is not at a near-tie ({tie_dist.max()})"
    assert q_gpu.min(initial=0) >= -127 and q_gpu.max(initial=0) <= 127, "a code outside the range [-127, 127]"
    return {"mismatch_frac": frac, "scale_rel_max": float(rel.max(initial=0.0))}


OUT_REL = {"bf16": 2.0**-8, "f16": 2.0**-11}  # half an ulp, relative: 8 and 11 significant bits
OUT_ABS = {"bf16": 2.0**-134, "f16": 2.0**-25}  # half the smallest subnormal
F32_REL = 2.0**-21                           # a few float32 roundings in the epilogue (2^-24 each)
GELU_REL = 4e-7                              # erf approximation (<= 1.5e-7) and exp rounding, relative to |z|


def check_output_elementwise(y: np.ndarray, acc: np.ndarray, s_x: np.ndarray, s_w, bias=None, addend=None,
                             gelu: bool = False, out: str = "bf16") -> float:
    """Bound every output element against z = acc * (s_x[m] * s_w) + bias[n] (+ addend), then GELU.

    ``acc``, ``s_x`` and ``s_w`` are the kernel's own int32 accumulators (from
    the oracle's exact GEMM of the kernel's codes) and scales, which the
    caller has already checked against the oracle with ``check_codes``. What
    is left between the kernel and this float64 value is the epilogue's
    float32 arithmetic and the single rounding to the output dtype:

        |y - ref| <= OUT_REL * |ref| + (1 + OUT_REL) * err + OUT_ABS,
        err = F32_REL * (|acc * s_x * s_w| + |bias| + |addend|)  (times 1.13, GELU's largest slope,
              plus GELU_REL * |z| with GELU).

    Returns the largest |y - ref| / bound (<= 1 passes); raises on a violation.
    """
    y = np.asarray(y, np.float64)
    acc = np.asarray(acc, np.float64)
    sx = np.asarray(s_x, np.float64)[:, None]
    sw = np.asarray(s_w, np.float64)
    sw = sw[None, :] if sw.ndim == 1 and sw.size > 1 else sw.reshape(())
    prod = acc * (sx * sw)
    z = prod.copy()
    mag = np.abs(prod)
    if bias is not None:
        b = np.asarray(bias, np.float64)[None, :]
        z = z + b
        mag = mag + np.abs(b)
    if addend is not None:
        a = np.asarray(addend, np.float64)
        z = z + a
        mag = mag + np.abs(a)
    err = F32_REL * mag
    if gelu:
        from scipy.special import erf

        ref = 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))
        err = 1.13 * err + GELU_REL * np.abs(z)
    else:
        ref = z
    bound = OUT_REL[out] * np.abs(ref) + (1.0 + OUT_REL[out]) * err + OUT_ABS[out] + 1e-300
    assert np.all(np.isfinite(y)), "a non-finite output element"
    ratio = np.abs(y - ref) / bound
    worst = float(ratio.max(initial=0.0))
    if worst > 1.0:
        i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(f"output element {tuple(int(v) for v in i)} = {y[i]!r}, expected {ref[i]!r} "
                             f"within {bound[i]:.3e} ({worst:.2f} x the bound)")
    return worst


def nrmse(y: np.ndarray, ref: np.ndarray) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / den) if den > 0 else float(np.linalg.norm(y))
