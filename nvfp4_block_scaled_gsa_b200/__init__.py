"""B200-native (sm_100a) NVFP4 Mixture-of-Experts expert-FFN.

The compute path is the C-ABI library ``_lib/libnvfp4moe.so`` (hand-written CUDA, declared in
``include/nvfp4_moe.h``); this package only builds it, loads it with ctypes and marshals torch
tensors and the current CUDA stream into its calls.
"""

from .api import (  # noqa: F401
    NVFP4Weights,
    ffn_workspace_bytes,
    gemm_dense,
    grouped_gemm,
    l1_swiglu_q,
    l1_swiglu_q_stats,
    l2_form,
    l2_scatter,
    l2_scatter_add,
    linear,
    linear_workspace_bytes,
    moe_ffn_forward,
    mxfp4_grouped_gemm,
    mxfp4_quantize,
    moe_ffn_forward_ex,
    permute,
    quantize,
    quantize_w1,
    quantize_weights,
    rmsnorm_quantize,
    scale_from_amax,
    w1_row_map,
    read_status,
    rows_max,
    sf_bytes,
    shared_expert,
    shared_expert_workspace_bytes,
)
from ._native import Nvfp4Error, lib  # noqa: F401
