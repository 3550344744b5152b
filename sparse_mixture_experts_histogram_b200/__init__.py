"""B200 (sm_100a) sparse Mixture-of-Experts feed-forward layer, forward pass.

The compute lives in the CUDA library ``libmoe_b200.so`` behind the C ABI of
``include/moe.h``; ``binding`` exposes the same entry points to Python.
``synth`` draws the seeded synthetic inputs and ``accounting`` holds the
FLOP/byte/parameter closed forms used for throughput and roofline numbers.
"""
from .binding import (  # noqa: F401
    ABI_FUNCTIONS,
    ACT_SIGMOID,
    ACT_SILU,
    WEIGHTS_ENTROPY,
    WEIGHTS_SIGMOID,
    WEIGHTS_SOFTMAX_ALL,
    WEIGHTS_SOFTMAX_TOPK,
    MoEError,
    MoEVariant,
    load_library,
    moe_combine,
    moe_ep_combine,
    moe_ep_dispatch,
    moe_ep_expert_ffn,
    moe_ep_ffn_splits,
    moe_ep_output_bf16,
    moe_ep_recv_rows,
    moe_ep_workspace_size,
    moe_expert_ffn,
    moe_expert_ffn_static,
    moe_expert_ffn_static_bytes,
    moe_expert_ffn_static_error,
    moe_forward,
    moe_forward_ex,
    moe_forward_fp8,
    moe_forward_fp8_traced,
    moe_forward_traced,
    moe_forward_variant,
    moe_get_device_error,
    moe_ipc_close,
    moe_ipc_get_handle,
    moe_ipc_open_handle,
    moe_permute,
    moe_route,
    moe_route_variant,
    moe_selftest_wait_timeout,
    moe_status_string,
    moe_workspace_size,
    moe_workspace_size_ex,
)
