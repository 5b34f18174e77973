"""B200 (sm_100a) sparse-MoE FFN layer: a C-ABI CUDA library (``libmoe_layer.so``,
declared in ``include/moe_layer.h``) and its thin Python binding.

    from sparse_moe_layer_warp_b200 import MoELayer
"""
from .binding import (  # noqa: F401
    EXPORTS,
    MOE_BF16,
    MOE_F32,
    MoEError,
    MoELayer,
    load_library,
    moe_config,
    moe_device_status,
    moe_forward,
    moe_forward_profiled,
    moe_forward_launch_count,
    moe_selftest_wait_timeout,
    moe_expert_health,
    moe_backward,
    moe_backward_workspace_size,
    MOE_PROFILE_STAGES,
    PROFILE_STAGE_NAMES,
    moe_layer_destroy,
    moe_layer_init,
    moe_route,
    moe_route_from_logits,
    moe_router_logits_static,
    moe_router_stats,
    moe_update_router_bias,
    moe_workspace_init,
    moe_workspace_size,
    status_string,
)
