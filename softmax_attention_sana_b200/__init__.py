"""B200-native (sm_100a) hot path of SANA-Video 2.0's hybrid linear-softmax attention.

The compute lives in libsana.so (C ABI declared in include/sana.h, kernels in
csrc/); this package is a thin ctypes binding over it.
"""

from ._lib import (EPI_NONE, EPI_RESIDUAL, EPI_SILU, Rope, SanaError, attnres_route,
                   attnres_route_bwd, check,
                   gemm_bf16, host_rope_tables, hybrid_stack_fwd, hybrid_stack_workspace_size,
                   hybrid_stack_workspace_views, last_error, lib,
                   linattn_apply, linattn_bwd, linattn_block_causal_scan, linattn_block_causal_scan_workspace_size,
                   linattn_block_causal_step, linattn_fwd, linattn_state,
                   linattn_workspace_size, mx_gemm, mx_linear, mx_quantize, mx_quantize_stack_weights,
                   rmsnorm, rope_apply,
                   softmax_anchor_rotated_fwd,
                   anchor_tile_count, softmax_anchor_fwd, softmax_anchor_sparse_fwd,
                   softmax_anchor_sparse_workspace_size, stack_config,
                   sync_status)

__all__ = [
    "EPI_NONE", "EPI_RESIDUAL", "EPI_SILU", "Rope", "SanaError", "attnres_route",
    "attnres_route_bwd", "check",
    "gemm_bf16", "host_rope_tables", "hybrid_stack_fwd", "hybrid_stack_workspace_size",
    "hybrid_stack_workspace_views", "last_error", "lib",
    "linattn_apply", "linattn_bwd", "linattn_block_causal_scan", "linattn_block_causal_scan_workspace_size",
    "linattn_block_causal_step", "linattn_fwd", "linattn_state", "linattn_workspace_size", "rmsnorm",
    "mx_gemm", "mx_linear", "mx_quantize", "mx_quantize_stack_weights", "rope_apply",
    "softmax_anchor_rotated_fwd",
    "anchor_tile_count", "softmax_anchor_fwd", "softmax_anchor_sparse_fwd",
    "softmax_anchor_sparse_workspace_size", "stack_config",
    "sync_status",
]
