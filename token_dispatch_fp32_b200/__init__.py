"""MoE routing hot path (router, dispatch, gather, combine) for NVIDIA B200.

The compute lives in libmr.so (hand-written sm_100a CUDA kernels behind the
C ABI in include/mr.h); this package is its thin Python binding.
"""
from ._binding import (  # noqa: F401
    MR_BF16, MR_ERR_CUDA, MR_ERR_DEVICE, MR_ERR_INVALID_ARG, MR_ERR_OVERFLOW, MR_ERR_TIMEOUT,
    MR_ERR_UNSUPPORTED, MR_F32, MR_MASK_NEG_INF, MR_MASK_ZERO, MR_OK, MR_PREC_3XTF32,
    MR_GROUP_MAX, MR_NORM_NO_EPS, MR_PREC_BF16X3, MR_PREC_FFMA, MR_PREC_TF32, MR_SCORE_SOFTMAX,
    MRError, lib, mr_combine, mr_dispatch, mr_ep_combine_p2p, mr_ep_dispatch_p2p,
    mr_ep_recv_order, mr_expert_gemm_gather, mr_ipc_close, mr_ipc_export, mr_ipc_import,
    mr_expert_gemm_gather_combine, mr_expert_gemm_gather_packed, mr_expert_pack_weights,
    mr_dispatch_noalloc, mr_dispatch_noalloc_max_workspace,
    mr_dispatch_workspace_size, mr_gather_rows, mr_get_error, mr_launch_count, mr_router_forward,
    mr_router_forward_bf16w, mr_router_forward_ex, mr_router_forward_max_scratch, mr_router_workspace_size,
    status_string, version)
