"""CPU oracle of the INT8 ConvRot linear layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the library never does.
"""

from .attention_oracle import (  # noqa: F401
    attention_exact,
    attention_int8,
    attention_logits,
    quantize_heads,
    softmax,
)
from .convrot_oracle import (  # noqa: F401
    QMAX,
    bf16_to_f64,
    dequant,
    dequant_per_channel,
    f16_to_f64,
    gelu_erf,
    gemm_s32,
    hadamard,
    linear,
    linear_ex,
    nrmse,
    prepare_weight,
    prepare_weight_per_channel,
    quant_act,
    quantize_per_token,
    quantize_tensorwise,
    rotate,
    rotation_matrix,
    to_bf16_rne,
    to_f16_rne,
)
