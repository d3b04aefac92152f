"""B200-native (sm_100a) routed Mixture-of-Experts FFN layer.

The public calls mirror the C ABI of include/moe.h:

    ids, weights = route(x, w_router, k, bias=None, renorm=True)
    y            = forward(x, w_router, w_gate, w_up, w_down, k, bias=None, renorm=True)
    g            = ForwardGraph(x, w_router, w_gate, w_up, w_down, k); y = g.replay()
    y_dense      = dense_ffn(x, w_gate_d, w_up_d, w_down_d)   # the dense MLP beside the MoE

x, weights and outputs are CUDA tensors (bf16 operands, int32 ids, fp32 routing weights);
all arithmetic runs in libmoe_b200.so.  ``workloads`` (seeded synthetic inputs) can be
imported without a GPU.
"""
from ._abi import (ForwardGraph, MoEError, dense_ffn, ffn_kernel_name, forward,  # noqa: F401
                   last_kernel_count, last_stage_times, load, route, router_stats, status_string,
                   sync_status)

__all__ = ["route", "forward", "dense_ffn", "ForwardGraph", "sync_status", "last_stage_times",
           "load", "router_stats", "status_string", "MoEError", "last_kernel_count",
           "ffn_kernel_name"]
