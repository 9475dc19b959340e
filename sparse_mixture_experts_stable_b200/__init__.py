"""Capacity-limited top-k sparse mixture-of-experts layer for NVIDIA B200 (sm_100a).

The computation lives in ``libmoe.so`` (C ABI, ``include/moe.h``); this package
holds the CUDA sources (``csrc/``), the build step (``build.py``), the ctypes
binding (``binding.py``), a layer helper that chains the entry points with
preallocated buffers (``layer.py``) and the seeded synthetic workloads
(``inputs.py``).
"""
from .binding import (  # noqa: F401
    EXPORTED, LIB_PATH, MoeError, lib, moe_aux_stats, moe_backward, moe_backward_gelu, moe_backward_swiglu,
    moe_capacity, moe_clear_status, moe_combine, moe_dispatch, moe_dispatch_static, moe_ep_combine, moe_ep_dispatch,
    moe_ep_plan, moe_expert_ffn, moe_expert_ffn_gathered, moe_expert_ffn_save, moe_ipc_close, moe_ipc_export, moe_ipc_import,
    moe_read_status, moe_renormalize_kept_gates, moe_route, moe_router_backward, moe_transpose_weights, new_status,
    status_string, moe_swiglu_layer_forward, moe_swiglu_layer_workspace_size, SwiGLULayerDesc,
)
