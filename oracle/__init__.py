"""CPU oracle for the W8A8 ConvRot expert-choice MoE block.

This package is TEST INFRASTRUCTURE. Only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it. The product path (the CUDA library and its Python
binding) never imports, links or executes anything in here, and nothing in
here imports the product package.

``lowbit_oracle`` defines the W4A8 / W6A8 weight formats (b-bit codes in the
rotated basis with an FP8 E4M3 scale per group of 16 and an FP32 scale per
row) and the linears and MoE block that read them.

Everything is plain NumPy: the rotation as an explicit fp64 Sylvester
Hadamard matrix, the quantiser's quotient in fp64, exact integer GEMMs, fp64
for the router softmax, fp32 for the scales, dequantised outputs, SwiGLU and
the router-weighted combine.
"""

from .convrot_oracle import (  # noqa: F401
    bf16_round,
    block_rotate,
    combine,
    combine_f32,
    dequant,
    down_from_codes,
    expert_choice_topc,
    hadamard,
    int_gemm,
    moe_block,
    quantize_rows,
    rotation_matrix,
    rotquant,
    router_softmax,
    silu_f32,
    swiglu_from_codes,
    w8a8_linear,
    w8a8_linear_from_codes,
)
from .lowbit_oracle import (  # noqa: F401
    dequant_weights_lowbit,
    e4m3_decode,
    e4m3_encode,
    lowbit_acc,
    lowbit_dequant,
    lowbit_linear,
    lowbit_linear_from_codes,
    lowbit_swiglu_from_codes,
    moe_block_lowbit,
    qmax_of,
    quantize_rows_lowbit,
    rotquant_lowbit,
)
