"""B200-native (sm_100a) forward pass of a Mixture-of-Experts FFN layer.

The layer runs in ``libmoe_b200.so`` (C ABI in ``include/moe.h``).  This package is the
thin Python binding: ``moe_route``, ``moe_permute``, ``moe_expert_ffn``, ``moe_combine``,
``moe_forward`` and ``moe_forward_host`` keep the C names and take torch CUDA tensors;
``MoELayer`` bundles a layer's weights and workspace; ``EPMoELayer`` is one rank of the
expert-parallel layer (experts spread over the ranks of a process group).  Accessing any of them loads the
library and raises ``ImportError`` if it has not been built -- there is no fallback.
"""
from __future__ import annotations

import importlib

from . import workloads  # noqa: F401  (seeded synthetic inputs; no layer arithmetic)

_NATIVE_NAMES = {
    "moe_workspace_size", "moe_workspace_init", "alloc_workspace", "moe_capacity", "moe_route",
    "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward", "moe_forward_host",
    "moe_check_status", "moe_last_launch_count", "moe_profile_begin", "moe_profile_end",
    "moe_route_static", "moe_forward_routed", "moe_route_hash", "moe_balance",
    "moe_permute_padded", "moe_forward_padded", "moe_forward_host_batches", "moe_config", "moe_route_out", "make_config",
    "config_from_shape", "MoeError", "lib", "EXPORTED", "moe_ep_first_expert", "moe_ep_plan",
    "moe_ep_workspace_size", "alloc_ep_workspace", "moe_permute_ep", "moe_ep_expert_ffn",
    "moe_ep_combine", "moe_ep_copy_runs", "moe_permute_ep_p2p", "moe_ep_combine_p2p",
    "ipc_handle", "ipc_open", "ipc_close",
}


def __getattr__(name):
    if name in _NATIVE_NAMES:
        return getattr(importlib.import_module("._native", __name__), name)
    if name == "MoELayer":
        return importlib.import_module(".layer", __name__).MoELayer
    if name == "EPMoELayer":
        return importlib.import_module(".ep", __name__).EPMoELayer
    raise AttributeError(name)
