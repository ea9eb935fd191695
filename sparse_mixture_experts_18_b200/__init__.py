"""B200 (sm_100a) forward pass of Mixtral's sparse Mixture-of-Experts block.

The computation lives in libmoe.so (hand-written CUDA kernels behind the C ABI declared in
include/moe.h); this package is its build script and a ctypes binding.
"""
from .moe import (MOE_BF16, MOE_F32, MoeError, alloc_workspace, lib, moe_forward,
                  moe_forward_debug, moe_forward_fp8, moe_forward_host_io,
                  moe_forward_noalloc, moe_forward_profiled, moe_plan_info,
                  moe_quantize_mx_e4m3, moe_stack_forward, moe_stack_workspace_bytes,
                  moe_workspace_bytes, moe_workspace_bytes_fp8, moe_workspace_status,
                  moe_noalloc_status, moe_stack_forward_profiled, moe_stack_forward_host_io,
                  moe_debug_forward_withheld, moe_route, moe_experts_forward, moe_combine,
                  moe_gather_rows)

__all__ = ["MOE_BF16", "MOE_F32", "MoeError", "alloc_workspace", "lib", "moe_forward",
           "moe_forward_debug", "moe_forward_fp8", "moe_forward_host_io",
           "moe_forward_noalloc", "moe_forward_profiled", "moe_plan_info",
           "moe_quantize_mx_e4m3", "moe_stack_forward", "moe_stack_workspace_bytes",
           "moe_workspace_bytes", "moe_workspace_bytes_fp8", "moe_workspace_status",
           "moe_noalloc_status", "moe_stack_forward_profiled", "moe_stack_forward_host_io",
           "moe_debug_forward_withheld", "moe_route", "moe_experts_forward", "moe_combine",
           "moe_gather_rows"]
