"""B200 (sm_100a) token-choice Mixture-of-Experts layer forward.

The computation lives in libmoe_b200.so (hand-written CUDA for sm_100a, C
ABI in include/moe.h). This package only builds it and marshals torch
tensors into its entry points:

    moe_route              router scores, softmax, top-k, gates
    moe_permute            per-expert counts/offsets, drops, dispatch permutation
    moe_pack_weights       gate/up interleave for the grouped FFN
    moe_grouped_ffn        grouped SwiGLU expert GEMMs over ragged groups
    moe_unpermute_combine  return outputs to their tokens, gate-weighted
    moe_layer_backward     gradients of the layer (moe_pack_weights_backward first)
    moe_layer_forward      all of the above on one stream (moe_layer_forward_timed
                           with stage events)
    moe_pack_weights_mxfp8 quantised expert weights for the MXFP8 grouped GEMMs
                           (config(..., precision="mxfp8"))
    moe_mxfp8_quantize     MXFP8 quantisation of a bf16 matrix along its rows
"""
from ._lib import (  # noqa: F401
    EXPORTED, LIB_PATH, MOE_DTYPE_BF16, MOE_DTYPE_F32, MOE_ERR_CUDA, MOE_ERR_INVALID_ARG, MOE_ERR_NO_DEVICE,
    MOE_DISPATCH_AUTO, MOE_DISPATCH_COPY, MOE_DISPATCH_GATHER, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE,
    MOE_EXPERT_IDENTITY, MOE_EXPERT_SCALE, MOE_EXPERT_SWIGLU,
    MOE_GEMM_TILES_AUTO, MOE_GEMM_TILES_PAIR, MOE_GEMM_TILES_SINGLE, MOE_LAYOUT_COMPACT, MOE_LAYOUT_PADDED,
    MOE_MAX_E, MOE_MAX_K, MOE_OK, MOE_OP_BACKWARD, MOE_OP_GROUPED_FFN, MOE_OP_LAYER, MOE_OP_PERMUTE, MOE_OP_ROUTE,
    MOE_PACK_BLOCK,
    MOE_COMBINE_AUTO, MOE_COMBINE_FUSED, MOE_COMBINE_SEPARATE, MOE_PREACT_RECOMPUTE, MOE_PREACT_SAVE, MOE_PRECISION_BF16, MOE_PRECISION_MXFP8, MOE_STATUS_MX_SATURATED, MOE_STATUS_MX_UNDERFLOW,
    MOE_STATUS_BAD_ROUTE, MOE_STATUS_NAN_LOGIT, MOE_STATUS_TIMEOUT, MoeConfig, MoeError, config, lib,
    moe_grouped_ffn, moe_layer_backward, moe_layer_forward, moe_pack_weights, moe_pack_weights_backward,
    moe_permute, moe_permute_static_scratch, moe_route,
    moe_unpermute_combine, moe_workspace_size, moe_gemm_tiles_used, perm_rows, workspace,
    moe_mxfp8_quantize, moe_mxfp8_weights_size, moe_pack_weights_mxfp8, mx_counters, mxfp8_scale_bytes)
