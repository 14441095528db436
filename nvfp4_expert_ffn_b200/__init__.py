"""NVFP4 mixture-of-experts layer forward for NVIDIA B200 (sm_100a).

The compute runs in libmoe_nvfp4.so (hand-written CUDA, C ABI in include/moe_nvfp4.h);
``binding`` marshals torch tensors into its calls, ``layer`` chains the calls for one
layer, ``synth`` draws seeded synthetic inputs.
"""
from .binding import (  # noqa: F401
    MOE_FFN_ACCUMULATE, MOE_FFN_PER_ASSIGN, MOE_OP_FFN, MOE_OP_LAYER, MOE_OP_QUANT, MOE_OP_ROUTE,
    MOE_PATH_AUTO, MOE_PATH_CUDA_CORE, MOE_PATH_DECODE, MOE_PATH_PREFILL, Experts, ExpertWeights, MoeError,
    moe_combine, moe_expert_ffn, moe_expert_hist, moe_get_device_status, moe_pack_experts,
    moe_permute, moe_route, moe_workspace_size, nvfp4_quantize_act)
