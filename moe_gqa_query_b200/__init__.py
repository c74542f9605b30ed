"""Grouped Query Experts (GQE) attention on NVIDIA B200 (sm_100a): forward and backward.

The computation lives in the CUDA library libgqe.so (C ABI in include/gqe.h);
this package is its thin Python binding plus GQELayer, which chains the calls.
Importing it without the built library raises ImportError: there is no CPU
fallback.
"""
from ._lib import (  # noqa: F401
    GQEError, gqe_dims, make_dims, header_functions, LIB_PATH,
    GQE_OP_ROUTED_QPROJ, GQE_OP_ATTN_DECODE, GQE_OP_COMBINE_OUT_PROJ, GQE_OP_ATTN_BWD,
    GQE_OP_LAYER_FORWARD, GQE_OP_LAYER_FORWARD_HOST, gqe_layer_weights, layer_weights,
    gqe_layer_forward, gqe_layer_forward_host,
    gqe_workspace_size, gqe_router_topk, gqe_router_stats, gqe_routed_qproj, gqe_kv_proj, gqe_kv_append,
    gqe_attn_prefill, gqe_attn_prefill_bwd, gqe_attn_decode, gqe_attn_decode_noalloc, DECODE_NOALLOC_MAX_BYTES, gqe_combine,
    gqe_combine_out_proj, gqe_linear, gqe_device_error, gqe_gemm, gqe_gemm_acc, gqe_combine_bwd, gqe_router_bwd, gqe_bwd_pack_cols,
    gqe_bwd_pack, gqe_bwd_pack_weights, gqe_transpose, gqe_transpose_f32,
    gqe_status_string, gqe_debug_exp2, gqe_debug_wait_timeout,
)
from .layer import GQEConfig, GQELayer  # noqa: F401
