"""B200 (sm_100a) W8A8 ConvRot expert-choice MoE: C-ABI CUDA library + binding.

The compute runs in libconvrot.so (built in-tree by ``build.py``); this
package only marshals arguments to it. Importing the package does not load
the library; the first call does, and raises if it is missing.
"""

from .binding import (  # noqa: F401
    ConvrotError,
    TiledWeights,
    LIB_PATH,
    convrot_check_device_error,
    convrot_combine_rows,
    convrot_count_wait_selftest,
    convrot_device_check,
    convrot_f32_to_bf16,
    convrot_gather_rows,
    convrot_i8_gemm_bf16,
    convrot_i8_gemm_i32,
    convrot_i8_gemm_scatter,
    convrot_i8_gemm_swiglu,
    convrot_i8_gemm_swiglu_rq,
    convrot_linear_workspace_size,
    convrot_quantize_weights,
    convrot_quantize_weights_tiled,
    convrot_rotquant,
    convrot_router_softmax,
    convrot_swiglu_rq_units,
    convrot_topc,
    convrot_wait_selftest,
    load_library,
    moe_expert_choice_forward,
    moe_stage_views,
    moe_workspace_layout,
    moe_workspace_size,
    quantize_moe_weights,
    tiled_weight_bytes,
    untile,
    w8a8_convrot_linear,
    w8a8_convrot_linear_noalloc,
)
