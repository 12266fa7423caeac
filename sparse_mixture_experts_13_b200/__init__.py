"""B200 (sm_100a) sparse mixture-of-experts layer: a C-ABI CUDA library
(``libmoe.so``, declared in include/moe.h) and its ctypes binding.

PyTorch serves only for device memory and streams; every step of the layer
(router, top-k gate, capacity, grouping, grouped SwiGLU GEMMs, combine) runs
in the library's kernels.
"""
from ._lib import (EXPORTED, MOE_ERR_BOUNDS, moe_debug_build, moe_debug_workspace_arm, moe_debug_workspace_check, MOE_DROP_BY_ORDER, MOE_DROP_BY_ORDER_NEXT_BEST, MOE_DROP_BY_PROB,
                   MOE_DROP_BY_PROB_NEXT_BEST, MOE_ERR_CUDA, MOE_ERR_INVALID_ARG,  # noqa: F401
                   MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_OK, MOE_VARIANT_AUTO,
                   MOE_VARIANT_STREAM, MOE_VARIANT_TILED, MOE_VARIANT_TILED_SINGLE, MoeError, check, lib, make_shape, moe_combine,
                   moe_grouped_swiglu, moe_layer_forward, moe_permute_noalloc, moe_permute_noalloc_status, moe_layer_forward_host,
                   moe_layer_forward_profiled, moe_permute,
                   moe_read_device_status, moe_router_topk, moe_selftest_wait_timeout, moe_shape, moe_workspace_size, status_string,
                   moe_quantize_q4, moe_workspace_size_q4, moe_grouped_swiglu_q4, moe_layer_forward_q4,
                   moe_layer_forward_q4_profiled, moe_layer_forward_q4_host, moe_router_stats, moe_ep_plan, moe_ep_dispatch, moe_ep_combine,
                   moe_ep_dispatch_cap, moe_ep_select, moe_ep_combine_cap)
from .layer import MoELayer, MoELayerQ4  # noqa: F401
