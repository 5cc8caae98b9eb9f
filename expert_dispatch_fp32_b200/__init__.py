"""Expert-parallel MoE-layer forward on one NVIDIA B200 (sm_100a).

The compute path is libmoe.so (hand-written CUDA behind a C ABI, include/moe.h);
this package holds its ctypes binding and a small layer object that allocates
buffers with PyTorch.  Stages, after "Expert Parallel (EP)", Communication
Pattern: moe_route -> moe_preprocess -> moe_dispatch_permute -> moe_expert_ffn
-> moe_combine_unpermute (moe_route_dispatch for the first three in one launch where
it applies, moe_forward for all five).
"""
from ._binding import (  # noqa: F401
    LIB_PATH, MOE_ACT_GELU, MOE_ACT_SWIGLU, MOE_DT_BF16, MOE_DT_F32, MOE_ERR_CUDA,
    MOE_ERR_INDEX_OOB, MOE_ERR_INVALID_ARG, MOE_ERR_SCRATCH_LIMIT, MOE_ERR_TIMEOUT,
    MOE_ERR_UNSUPPORTED, MOE_OK,
    MoeConfig, MoeEpPeers, MoeError, lib, moe_abi_version, moe_check_wait_timeout,
    moe_combine_unpermute, moe_dispatch_mxfp8, moe_dispatch_permute,
    moe_ep_local_ids, moe_ep_recv_layout, moe_ep_return_rows, moe_ep_send_counts, moe_ep_send_rows,
    moe_ipc_close, moe_ipc_export, moe_ipc_handle_bytes, moe_ipc_import, moe_instr_read,
    moe_ep_wait_returned, moe_ep_expert_ffn_return, moe_expert_ffn_mxfp8, moe_mxfp8_quantize, moe_packed_weights_mxfp8_size,
    moe_prepare_weights_mxfp8, moe_workspace_mxfp8_size, moe_expert_ffn, moe_forward, moe_gather_rows, moe_packed_weights_size,
    moe_prepare_weights, moe_preprocess, moe_preprocess_noalloc, moe_shared_ffn,
    moe_route, moe_route_dispatch, moe_route_dispatch_is_fused, moe_router_filter_view,
    moe_status_string, moe_validate_config, moe_workspace_size,
)
from .layer import MoELayer, make_config  # noqa: F401
