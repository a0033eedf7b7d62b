"""B200 (sm_100a) Mixtral sparse-MoE feed-forward layer: y = sum over the top-2 of
softmax(x W_g) of SwiGLU_i(x), E = 8 experts, k = 2 per token.

The compute lives in libmoe.so (hand-written CUDA kernels behind the C ABI of
include/moe.h); `binding` is a thin ctypes layer with the same function names.
Build the library with `python -m sparse_mixture_experts_05_b200.build`.
"""
from .binding import (  # noqa: F401
    EXPORTS, MOE_ERR_CUDA, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED,
    MOE_ERR_WORKSPACE, MOE_OK, MoeError, moe_aux_loss, moe_block_forward,
    moe_block_workspace_bytes, moe_check_shape, moe_combine, moe_dispatch, moe_expert_swiglu,
    moe_expert_swiglu_bias, moe_expert_swiglu_stall_test, moe_expert_workspace_bytes, moe_forward,
    moe_forward_bias, moe_forward_hostio, moe_forward_hostio_batches,
    moe_forward_hostio_batches_stall_test, moe_forward_hostio_batches_workspace_bytes,
    moe_forward_hostio_stall_test,
    moe_forward_hostio_workspace_bytes,
    moe_forward_kernel_count, moe_forward_profiled, moe_forward_static,
    moe_forward_workspace_bytes,
    moe_read_device_status, moe_route, status_string, workspace,
)
