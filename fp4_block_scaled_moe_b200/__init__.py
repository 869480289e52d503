"""fp4moe for B200: the routed-expert MoE layer on 4-bit block-scaled weights.

The computation lives in the CUDA library ``libfp4moe.so`` (C ABI, include/fp4moe.h);
this package only marshals torch tensors into it.
"""
from .api import (  # noqa: F401
    MoEWeights,
    alloc_workspace,
    fp4_f32_to_bf16,
    fp4_launch_count,
    fp4_linear,
    fp4_mma_scales,
    fp4_nvfp4_mma_scales,
    fp4_pack,
    fp4_pack_cb4,
    fp4_pack_v2a,
    fp4_unpack,
    fp4_unpack_v2a,
    fp4_workspace_kernel_stats,
    fp4_workspace_status,
    moe_fp4_forward,
    moe_fp4_expert_kernels,
    moe_fp4_forward_noalloc,
    moe_fp4_forward_partial,
    moe_fp4_noalloc_status,
    moe_fp4_workspace_size,
    moe_route,
    prepare_mma_scales,
)

__version__ = "0.1.0"
