"""Oracle jobs the GPU tests hand to spawned worker processes.

Plain CPU work (input generation and the fp64 oracle) with no CUDA and no
torch, so that a process pool started with ``spawn`` can run it while the
test process drives the GPU.
"""
import math

import numpy as np

import oracle as O
import synth
from synth.video_latents import round_to


def stack_layer_selection(layer, tau, heads):
    """The 75600-token stack's layer ``layer`` (mode = layer mod 3, per-head
    gains): bf16-rounded q, k of the given heads (float32 arrays) and, per
    head, the oracle's pair set and the 1e-4 relative band around its cut
    score (both bit-packed), and the oracle's k*."""
    w = synth.WORKLOADS[5]
    mode = layer % 3
    scale = 1.0 / math.sqrt(w.head_dim)
    q, k, _ = synth.make_qkv(w.wid, layer, w.T, w.H, w.W, max(heads) + 1, w.head_dim,
                             kind=w.kind, head_gain=w.head_gain)
    q, k = (round_to(x[:, list(heads)], "bf16") for x in (q, k))
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    S = O.block_scores(q, O.pool_blocks(k, w.T, w.H, w.W, box), scale)
    masks, bands, ks = [], [], []
    for i in range(len(heads)):
        m, st = O.threshold_select(S[i], tau)
        cut = st["cut_score"]
        masks.append(np.packbits(m))
        bands.append(np.packbits(np.abs(S[i] - cut) <= 1e-4 * abs(cut)))
        ks.append(st["k"])
    return layer, q.astype(np.float32), k.astype(np.float32), masks, bands, ks
