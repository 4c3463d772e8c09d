"""Sparse MoE FFN layer forward and backward on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libmoe_b200.so`` (declared in
``include/moe_b200.h``); this package is its Python binding: ctypes
declarations of the same entry points plus small helpers that turn torch
tensors into the pointers and structs the ABI takes.  PyTorch only provides
device memory and streams here.  There is no fallback: if the library is
missing or fails to load, importing the binding raises.
"""
from .abi import (  # noqa: F401
    LIB_PATH, MoEError, LayerDesc, Weights, WsLayout, lib,
    moe_status_string, moe_version, moe_device_status,
    moe_route_workspace_size, moe_route_topk,
    moe_permute_workspace_size, moe_permute, moe_permute_static_scratch,
    moe_expert_ffn_workspace_size, moe_expert_ffn,
    moe_shared_expert_workspace_size, moe_shared_expert,
    moe_combine, moe_workspace_size, moe_workspace_layout, moe_forward,
    moe_forward_profiled, moe_forward_launch_count, NUM_STAGE_EVENTS, STAGE_NAMES,
    moe_algorithmic_work, EXPORTED_SYMBOLS, moe_forward_add,
    DenseDesc, moe_dense_ffn_workspace_size, moe_dense_ffn, moe_dense_ffn_profiled, NUM_DENSE_EVENTS,
    Grads, moe_backward_workspace_size, moe_backward, moe_backward_launch_count, moe_gather_rows,
    moe_capacity_drop, moe_expert_capacity, moe_selftest_wait_timeout, moe_ep_pack, moe_ep_unpack,
    DTYPE_F32, DTYPE_BF16, GATE_SOFTMAX, GATE_SIGMOID_BIAS, ACT_GELU_TANH, ACT_SWIGLU,
    DEVERR_NONE, DEVERR_BAD_EXPERT_INDEX, DEVERR_TIMEOUT, DEVERR_BAD_ROW_TOKEN, DEVERR_BAD_COUNT,
)
from .layer import DenseLayer, MoELayer, dense_desc_from_config, desc_from_config, weights_from_tensors  # noqa: F401,E501
