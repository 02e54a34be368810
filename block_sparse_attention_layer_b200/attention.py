"""Caller-side glue around the VMoBA kernels: an autograd function over the C
ABI's forward / backward, and a self-attention module that places VMoBA where
a video DiT has full self-attention.

VMoBA notes, overall framework: VMoBA replaces the attention computation
itself (same input and output shapes as full attention); key design 1: layer
l partitions keys by mode l mod 3; training strategy: tau = 0.25, and the
first 25 % of denoising steps keep full attention.  The projections are plain
GEMMs (``torch.nn.Linear``); every attention step -- partition, pooling,
scores, selection, attention forward and backward -- runs in libvmoba.
"""
from __future__ import annotations

import math

import torch

from . import _lib
from ._lib import LayerShape
from .layer import VMoBALayer


class VMoBAFunction(torch.autograd.Function):
    """O = VMoBA(q, k, v) with the selection held constant for the backward
    (the selection is piecewise constant: no gradient flows through it).

    q, k, v: [s][n_heads][head_dim] contiguous CUDA tensors of the layer's
    dtype.  ``full`` selects every pair (dense attention over the blocks).

    The backward kernels read state the forward left in the layer's buffers
    (permuted keys and values, pair lists, LSE, the fp32 output copy).  Each
    call keeps its own selection bitmap and records the layer's forward
    generation; if another forward ran on the same layer in between (two
    micro-batches, activation checkpointing, a full-attention call), the
    backward first restores this call's state by re-running partition, plan
    and forward on its saved inputs and selection -- the same deterministic
    kernels, so the restored state is bit-identical -- and then runs.
    """

    @staticmethod
    def forward(ctx, q, k, v, layer: VMoBALayer, tau: float, full: bool, scale: float):
        if full:
            nb = layer.n_blocks
            bits = torch.full_like(layer.sel, -1)
            rem = nb % 32
            if rem:
                bits[..., -1] = (1 << rem) - 1
            layer.partition_only(k, v)
            layer.use_selection(bits)
        else:
            layer.select(q, k, v, tau, scale)
        out, _ = layer.forward(q, scale)
        ctx.layer, ctx.scale = layer, scale
        ctx.generation = layer.generation
        ctx.save_for_backward(q, k, v, layer.sel.clone())
        return out.clone()

    @staticmethod
    def backward(ctx, dout):
        q, k, v, sel = ctx.saved_tensors
        layer = ctx.layer
        if layer.generation != ctx.generation:
            # another forward replaced this call's state: rebuild it
            layer.partition_only(k, v)
            layer.use_selection(sel)
            layer.forward(q, ctx.scale)
            ctx.generation = layer.generation
        dq, dk, dv = layer.backward(q, dout.contiguous(), ctx.scale)
        return dq.clone(), dk.clone(), dv.clone(), None, None, None, None


class VMoBASelfAttention(torch.nn.Module):
    """Self-attention of one DiT layer over a (T, H, W) video latent with
    VMoBA in place of full attention.

    x: [s][dim] tokens in (t, y, x) order -> [s][dim].  ``boxes`` gives the
    (bt, bh, bw) box of each partition mode (mode = layer_idx mod 3);
    ``full_attention=True`` in ``forward`` keeps every pair (the early
    denoising steps of the training strategy).
    """

    def __init__(self, dim: int, n_heads: int, T: int, H: int, W: int, layer_idx: int,
                 boxes, tau: float = 0.25, dtype=torch.bfloat16, device="cuda"):
        super().__init__()
        if dim % n_heads:
            raise ValueError("dim must be a multiple of n_heads")
        self.n_heads, self.head_dim = n_heads, dim // n_heads
        self.mode = _lib.mode_for_layer(layer_idx)
        self.tau = float(tau)
        self.qkv = torch.nn.Linear(dim, 3 * dim, bias=True, device=device, dtype=dtype)
        self.proj = torch.nn.Linear(dim, dim, bias=True, device=device, dtype=dtype)
        bt, bh, bw = boxes[self.mode]
        dt = "bf16" if dtype == torch.bfloat16 else "f32"
        self.shape = LayerShape(T, H, W, n_heads, self.head_dim, self.mode, bt, bh, bw, dt)
        self.layer = VMoBALayer(self.shape, device=device)
        self.scale = 1.0 / math.sqrt(self.head_dim)

    def forward(self, x: torch.Tensor, full_attention: bool = False) -> torch.Tensor:
        s = x.shape[0]
        qkv = self.qkv(x).view(s, 3, self.n_heads, self.head_dim)
        q, k, v = (qkv[:, i].contiguous() for i in range(3))
        o = VMoBAFunction.apply(q, k, v, self.layer, self.tau, bool(full_attention), self.scale)
        return self.proj(o.reshape(s, self.n_heads * self.head_dim))


def full_attention_steps(n_steps: int, fraction: float = 0.25) -> int:
    """Denoising steps (from the first) that keep full attention: the notes'
    training strategy keeps it for the first 25 % of steps."""
    return int(math.ceil(fraction * n_steps))
