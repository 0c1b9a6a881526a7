"""B200 (sm_100a) OLMoE mixture-of-experts FFN layer.

The compute lives in libmoe_b200.so (C ABI in include/moe.h); `binding`
marshals torch tensors into it under the same function names, and
`synthetic` draws seeded inputs with OLMoE's shapes.
"""

from .binding import (  # noqa: F401
    EXPORTS,
    MOE_BF16,
    MOE_FP32,
    ROW_ALIGN,
    MoeError,
    MoELayer,
    config,
    grad_torch_dtype,
    lib,
    moe_backward,
    moe_check_config,
    moe_combine,
    moe_combine_residual,
    moe_dispatch,
    moe_expert_choice_capacity,
    moe_expert_down,
    moe_expert_ffn,
    moe_expert_gate_up,
    moe_forward,
    moe_forward_decode,
    moe_forward_expert_choice,
    moe_forward_host,
    moe_forward_host_async,
    moe_get_device_status,
    moe_padded_rows,
    moe_rmsnorm,
    moe_route,
    moe_route_expert_choice,
    moe_route_static,
    moe_set_stage_events,
    moe_stack_forward,
    moe_stack_forward_trace,
    moe_workspace_bytes,
    moe_workspace_init,
    status_string,
    torch_dtype,
    workspace,
)
