"""B200-native (sm_100a) DoRA factored row norm and fused compose.

``factored_weight_norm_b200.dora`` is the Python binding of libdora.so; the
computation itself runs in the library's CUDA kernels.
"""

from .dora import (  # noqa: F401
    DoraError,
    dora_compose_bwd,
    dora_compose_bwd_workspace_size,
    dora_compose_fwd,
    dora_device_status,
    dora_factored_norm,
    dora_factored_norm_workspace_size,
    dora_num_sms,
    dora_status_string,
)
