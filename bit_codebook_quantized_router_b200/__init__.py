"""B200-native routed-expert MoE feed-forward over 4-bit codebook weights.

The compute lives in ``libmoe_q4.so`` (hand-written sm_100a CUDA kernels
behind a C ABI, declared in ``include/moe_q4.h``); this package is a thin
binding.  Importing it does not load the library; the first call does, and
raises if the library was not built (there is no CPU fallback).
"""
from ._lib import (Layer, MoeQ4Error, Shared, alloc_workspace, combine, dequant, forward, forward_ex,
                   forward_ex_workspace, forward_gated, forward_gated_workspace, forward_host, forward_host_async,
                   forward_host_workspace, forward_stages, forward_status, forward_workspace, lib, lloyd_fit, pack,
                   route, router, router_workspace, status_string)

__all__ = ["Layer", "MoeQ4Error", "Shared", "alloc_workspace", "combine", "dequant", "forward", "forward_ex",
           "forward_ex_workspace", "forward_gated", "forward_gated_workspace", "forward_host", "forward_host_async",
           "forward_host_workspace", "forward_stages", "forward_status", "forward_workspace", "lib", "lloyd_fit",
           "pack", "route", "router", "router_workspace", "status_string"]
