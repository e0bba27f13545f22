"""B200-native forward and backward passes of a DeepSeek-style fine-grained mixture-of-experts
FFN layer, with an fp8 (E4M3) storage of the low-rank experts.

The compute path is the sm_100a CUDA library ``lib/libmoe.so`` behind the C ABI in
``include/moe.h``; :mod:`.binding` marshals arguments to it and :class:`MoELayer` holds device
weights and a workspace. The library is loaded lazily and there is no fallback path: without
the built library every call raises.
"""
from .binding import (DEBUG_FORCE_EXACT, DEBUG_PROFILE, DEBUG_WAIT_LIMIT_NS, EXPORTED,  # noqa: F401
                      MoEConfig, MoEError, MoEWeights, load, make_config, make_weights,
                      moe_aux_loss, moe_bias_update, moe_capacity, moe_combine,
                      moe_combine_backward, moe_debug_set, moe_route_backward,
                      moe_expert_backward, moe_backward_workspace_size, make_grads,
                      moe_debug_wait_timeout_probe, moe_expert_forward, moe_get_device_error,
                      moe_layer_forward, moe_permute, moe_profile_read, moe_quantize_fp8,
                      moe_route, moe_route_noalloc, moe_workspace_size, status_str)
from .layer import (MoELayer, quantize_lowrank_weights, torch_dtype, upload_weights,  # noqa: F401
                    y_perm_dtype)
