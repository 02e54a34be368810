"""Per-layer driver over the C ABI: owns the buffers of one VMoBA layer.

A thin convenience around ``_lib``: it allocates the caller-side buffers
with PyTorch (device memory only) and issues the ABI calls in order
partition -> score_select -> build_plan -> attn_fwd [-> attn_bwd] on the
current CUDA stream.  All arithmetic runs in libvmoba's kernels.
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import LayerShape


class VMoBALayer:
    """Buffers + calls for one layer shape (reusable across steps)."""

    def __init__(self, shape: LayerShape, device="cuda", max_pair_fraction=None):
        """max_pair_fraction: size the workspace for selections keeping at
        most that share of each head's pairs (tau for the method's threshold
        selection); None sizes it for every pair."""
        self.shape = shape
        s, h, d = shape.s, shape.n_heads, shape.head_dim
        dt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
        self.dtype = dt
        nb = _lib.num_blocks(shape)
        self.n_blocks = nb
        self.block_len = shape.s // nb
        dev = torch.device(device)
        self.k_perm = torch.empty((h, s, d), dtype=dt, device=dev)
        self.v_perm = torch.empty((h, s, d), dtype=dt, device=dev)
        self.blocks = torch.empty((h, nb, d), dtype=torch.float32, device=dev)
        self.sel = torch.empty((h, s, (nb + 31) // 32), dtype=torch.int32, device=dev)
        self.stats = torch.empty((h * _lib.HEAD_STATS_DTYPE.itemsize,), dtype=torch.uint8,
                                 device=dev)
        self.ws = torch.empty((_lib.workspace_size(shape, max_pair_fraction),), dtype=torch.uint8,
                              device=dev)
        self.ws_bwd = torch.empty((_lib.bwd_workspace_size(shape),), dtype=torch.uint8,
                                  device=dev)
        self.out = torch.empty((s, h, d), dtype=dt, device=dev)
        self.lse = torch.empty((h, s), dtype=torch.float32, device=dev)
        self.dq = torch.empty((s, h, d), dtype=dt, device=dev)
        self.dk = torch.empty((s, h, d), dtype=dt, device=dev)
        self.dv = torch.empty((s, h, d), dtype=dt, device=dev)
        # forwards run so far: lets a caller tell whether the forward state in
        # the buffers (LSE, fp32 output copy, pair lists) is still its own
        self.generation = 0

    def select(self, q, k, v, tau, scale=0.0):
        sh = self.shape
        _lib.partition(sh, k, v, self.k_perm, self.v_perm, self.blocks)
        _lib.score_select(sh, q, self.blocks, tau, scale, self.sel, self.stats, self.ws)
        _lib.build_plan(sh, self.sel, self.ws)

    def select_variant(self, q, k, v, variant, param, scale=0.0):
        """As select, with one of the ablation's selection rules (see
        _lib.score_select_variant): "threshold_global" (the method),
        "topk_global", "threshold_local", "topk_local"."""
        sh = self.shape
        _lib.partition(sh, k, v, self.k_perm, self.v_perm, self.blocks)
        _lib.score_select_variant(sh, q, self.blocks, variant, param, scale, self.sel,
                                  self.stats, self.ws)
        _lib.build_plan(sh, self.sel, self.ws)

    def use_selection(self, sel_bits):
        """Adopt a caller-built bitmap (e.g. a reference selection) and plan for it."""
        self.sel.copy_(sel_bits)
        _lib.build_plan(self.shape, self.sel, self.ws)

    def partition_only(self, k, v):
        _lib.partition(self.shape, k, v, self.k_perm, self.v_perm, self.blocks)

    def forward(self, q, scale=0.0):
        _lib.attn_fwd(self.shape, q, self.k_perm, self.v_perm, self.sel, self.ws, scale,
                      self.out, self.lse)
        self.generation += 1
        return self.out, self.lse

    def backward(self, q, dout, scale=0.0):
        _lib.attn_bwd(self.shape, q, self.k_perm, self.v_perm, self.sel, self.ws, scale,
                      self.lse, dout, self.dq, self.dk, self.dv, self.ws_bwd)
        return self.dq, self.dk, self.dv

    def step(self, q, k, v, tau, dout=None, scale=0.0):
        """One layer: partition, select, plan, forward (and backward if dout)."""
        self.select(q, k, v, tau, scale)
        self.forward(q, scale)
        if dout is not None:
            self.backward(q, dout, scale)

    def head_stats(self):
        return _lib.decode_stats(self.stats)
