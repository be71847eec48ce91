"""Plant plausible mistakes in a copy of the oracle and check that its pins catch each one.

The copy lives in a temporary directory; the real oracle is never modified.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "dropped_inv_sqrt_g": ("(blocks @ (hadamard(g) / np.sqrt(g)))", "(blocks @ hadamard(g))"),
    "round_half_up": ("q = np.rint(xr / safe[..., None])", "q = np.floor(xr / safe[..., None] + 0.5)"),
    "per_tensor_activation_scale": ("amax = np.max(np.abs(xr), axis=-1)",
                                    "amax = np.max(np.abs(xr)) + 0 * np.max(np.abs(xr), axis=-1)"),
    "bias_dropped": ("y = y + np.asarray(bias, np.float64)[None, :]", "y = y"),
    "qmax_128": ("QMAX = 127", "QMAX = 128"),
    "weight_scale_dropped": ("(np.asarray(s_x, np.float64)[:, None] * np.float64(s_w))",
                             "(np.asarray(s_x, np.float64)[:, None])"),
    "strided_instead_of_contiguous_groups": (
        "blocks = x.reshape(x.shape[:-1] + (K // g, g))",
        "blocks = x.reshape(x.shape[:-1] + (g, K // g)).swapaxes(-1, -2)"),
    "weight_columns_reversed": ("np.asarray(wq, np.float64).T", "np.asarray(wq, np.float64)[:, ::-1].T"),
    "token_scale_not_float32": ("s = (amax / QMAX).astype(np.float32)", "s = (amax / QMAX)"),
    "gelu_tanh_approximation": ("return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))",
                                "return 0.5 * y * (1.0 + np.tanh(0.7978845608028654 * (y + 0.044715 * y**3)))"),
    "f16_read_as_bf16": ("return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)",
                         "return bf16_to_f64(bits)"),
    "per_channel_scale_tensorwise": ("    return quantize_per_token(rotate(w, g))\n",
                                     "    q, s = quantize_tensorwise(rotate(w, g))\n    return q, np.full(q.shape[0], s)\n"),
    "addend_dropped": ("        y = y + np.asarray(addend, np.float64)\n", "        y = y\n"),
    "bf16_low_mantissa_dropped": ("(np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16)",
                                  "((np.asarray(bits, dtype=np.uint16).astype(np.uint32) & 0xFFF0) << 16)"),
    "per_channel_scale_on_tokens_axis": ("np.asarray(s_w, np.float64)[None, :])", "np.asarray(s_w, np.float64)[:, None])"),
}


# mistakes planted in the attention oracle, caught by its own pins
MUTATIONS_ATTENTION = {
    "softmax_scale_dropped": ("        * np.float64(softmax_scale)", "        * 1.0"),
    "keys_not_rotated": ("    kc, sk = quantize_heads(k, g)", "    kc, sk = quantize_per_token(np.asarray(k, np.float64))"),
    "softmax_over_queries": ("    m = np.max(s, axis=-1, keepdims=True)\n    e = np.exp(s - m)\n    return e / np.sum(e, axis=-1, keepdims=True)",
                             "    m = np.max(s, axis=-2, keepdims=True)\n    e = np.exp(s - m)\n    return e / np.sum(e, axis=-2, keepdims=True)"),
    "probabilities_not_normalised": ("    return e / np.sum(e, axis=-1, keepdims=True)", "    return e"),
    "key_scale_dropped": ("np.asarray(sk, np.float64)[..., None, :]) \\", "1.0) \\"),
}


def _run_mutated(tmp_path, file_name, old, new, test_file):
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    path = tmp_path / "oracle" / file_name
    src = path.read_text()
    assert old in src, "mutation target not found: the oracle changed, update this table"
    path.write_text(src.replace(old, new))
    return subprocess.run([sys.executable, "-m", "pytest", test_file, "-q", "-x"],
                          cwd=tmp_path, capture_output=True, text=True, timeout=300)


@pytest.mark.parametrize("name", sorted(MUTATIONS_ATTENTION))
def test_attention_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS_ATTENTION[name]
    r = _run_mutated(tmp_path, "attention_oracle.py", old, new, "tests/test_oracle_attention.py")
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    path = tmp_path / "oracle" / "convrot_oracle.py"
    src = path.read_text()
    assert old in src, "mutation target not found: the oracle changed, update this table"
    path.write_text(src.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle.py", "-q", "-x"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
