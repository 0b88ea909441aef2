"""B200 (sm_100a) forward pass of a top-k routed MoE FFN layer.

The computation lives in libmoe.so (C ABI declared in include/moe.h); this
package is its binding.  Importing it loads the library, so a missing or
unloadable library is an import error -- there is no other code path.
"""

from . import _abi
from ._abi import (  # noqa: F401
    EXPORTED, MOE_BF16, MOE_ERR_CUDA, MOE_ERR_DEVICE_BOUNDS, MOE_ERR_INVALID_ARG, MOE_ERR_TIMEOUT,
    MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_EXPERT_ATOMIC_GELU, MOE_EXPERT_SWIGLU, MOE_F32, MOE_OK,
    MoEError, MoELayerDesc, MoELayerWeights, moe_combine, moe_get_device_status, moe_grouped_ffn,
    moe_grouped_ffn_phase, moe_last_launch_count, moe_layer_forward, moe_layer_forward_host,
    moe_layer_host_workspace_size, moe_layer_workspace_size, moe_num_groups, moe_permute, moe_permute_static,
    moe_ep_expert_range, moe_ep_owner, moe_ep_plan, moe_fused_ffn_combine, moe_fused_workspace_size, moe_route, moe_row_capacity, moe_selftest_wait_timeout,
    moe_workspace_size, status_string, weights_struct)
from .layer import (MoELayer, StageBuffers, desc_from, make_desc, out_dtype, run_stages,  # noqa: F401
                    torch_dtype)

lib = _abi.load()
