"""MXFP4 MoE block-verify on B200: a C-ABI CUDA library with a thin binding.

The six calls of the verify step -- moe_route_topk, moe_permute,
mxfp4_moe_ffn, moe_combine, block_accept_greedy, block_accept_rejection --
plus moe_route_permute (the first two in one launch), moe_rms_norm for
stacked layers, the bonus-row acceptance variants and the MXFP4 weight
quantiser, all run as hand-written sm_100a
kernels in libmxfp4_moe.so (see include/mxfp4_moe.h).  Importing the package
does not load the library; the first call does, and raises if it is missing.
"""
from ._lib import (  # noqa: F401
    DEV_BAD_EXPERT, DEV_BAD_INDEX, DEV_BAD_TOKEN, DEV_NO_MASS, DEV_OK, DEV_TIMEOUT,
    FFN_AUTO, FFN_FMA, FFN_TENSOR, FFN_TENSOR_F4, FFN_TENSOR_F8, FFN_TENSOR_F8_PAIR, FFN_TENSOR_FUSED, MoeError, alloc_workspace, block_accept_greedy,
    block_accept_greedy_bonus, block_accept_rejection, block_accept_rejection_bonus, lib, moe_clear_device_status, moe_combine, moe_get_device_status,
    moe_permute, moe_rms_norm, moe_route_permute, moe_set_wait_limit_ns, moe_route_topk, mxfp4_moe_ffn, mxfp4_moe_ffn_noalloc,
    mxfp4_moe_ffn_workspace_bytes, mxfp4_quantize,
    workspace_h,
)
