"""B200-native VMoBA per-layer block-sparse attention.

The compute path is libvmoba.so (CUDA, sm_100a) behind the C ABI declared in
include/vmoba.h; this package is its Python binding (``_lib``), a buffer-
owning per-layer driver (``layer``), the in-tree build script (``build``) and
the bench's FLOP-count convention (``metrics``) and the split of a layer's
heads across GPUs (``sharding``).  Importing the package does
not load the library; the first ABI call does, and raises if it is missing.
"""
from ._lib import (  # noqa: F401
    LayerShape, VmobaError, lib, mode_for_layer, num_blocks, workspace_size,
    bwd_workspace_size, partition, score_select, build_plan, attn_fwd, attn_bwd, get_status,
    decode_stats, default_scale, kernel_launches, trace_enable, trace_read, score_select_static,
    score_select_variant, SELECT_VARIANTS, HEAD_STATS_DTYPE,
)

__all__ = [
    "LayerShape", "VmobaError", "lib", "mode_for_layer", "num_blocks", "workspace_size",
    "bwd_workspace_size", "partition", "score_select", "build_plan", "attn_fwd", "attn_bwd",
    "get_status", "decode_stats", "default_scale", "kernel_launches", "trace_enable", "trace_read",
    "score_select_static", "score_select_variant", "SELECT_VARIANTS", "HEAD_STATS_DTYPE",
]
