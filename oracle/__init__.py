"""CPU oracle of the INT8 ConvRot linear layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the library never does.
"""

from .convrot_oracle import (  # noqa: F401
    QMAX,
    bf16_to_f64,
    dequant,
    gemm_s32,
    hadamard,
    linear,
    nrmse,
    prepare_weight,
    quant_act,
    quantize_per_token,
    quantize_tensorwise,
    rotate,
    rotation_matrix,
    to_bf16_rne,
)
