"""B200-native (sm_100a) DoRA factored row norm, fused compose and their relatives.

``factored_weight_norm_b200.dora`` is the Python binding of libdora.so; the
computation itself runs in the library's CUDA kernels.
``factored_weight_norm_b200.sharded`` adds the one exchange a row-parallel
layer's norm needs.
"""

from .dora import (  # noqa: F401
    DoraError,
    dora_compose_bwd,
    dora_compose_bwd_noalloc,
    dora_compose_bwd_workspace_size,
    dora_compose_fwd,
    dora_device_status,
    dora_factored_norm,
    dora_factored_norm_batched,
    dora_factored_norm_batched_workspace_size,
    dora_factored_norm_bwd,
    dora_factored_norm_bwd_workspace_size,
    dora_factored_norm_sq,
    dora_factored_norm_workspace_size,
    dora_fused_linear_fwd,
    dora_fused_linear_fwd_workspace_size,
    dora_launch_count,
    dora_norm_finish,
    dora_num_sms,
    dora_status_string,
)
