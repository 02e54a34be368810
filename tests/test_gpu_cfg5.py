"""The 75600-token, 30-layer stack (T21 H45 W80, 12 heads with per-head Q/K
gains) on the tensor-core path, against the fp64 oracle.

Its blocks are 3600 / 1512 / 216 tokens (1D / 2D / 3D), so every mode ends
each block with a partial key chunk (16, 104 and 88 keys).  Layers of all
three modes are run at each of the stack's three thresholds with two heads
(heads are independent: per-head sizes and block shapes are the stack's); the
full pair set of each head is compared with the oracle's, then the heads
attend the oracle's own pairs and the outputs are compared on sampled query
rows.  The backward is checked at tau 0.25 on one layer of each mode.
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from synth.video_latents import round_to

from . import oracle_jobs
from .gpu_util import (TOL, from_device, out_err, pack_bits, pair_set_mismatch, sample_rows,
                       to_device, unpack_bits)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape  # noqa: E402
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402

W5 = synth.WORKLOADS[5]
SCALE = 1 / math.sqrt(W5.head_dim)
NH = 2
HEADS = (0, 1)


def _layer_inputs(layer, with_dout=False):
    w = W5
    q, k, v = synth.make_qkv(w.wid, layer, w.T, w.H, w.W, NH, w.head_dim, kind=w.kind,
                             head_gain=w.head_gain)
    out = [round_to(x, "bf16") for x in (q, k, v)]
    if with_dout:
        out.append(round_to(synth.make_dout(w.wid, layer, w.s, NH, w.head_dim), "bf16"))
    return out


def _select_and_pin(layer, tau, q, k, v):
    """GPU selection on all heads; the checked heads' pair sets must match the
    oracle's and are then replaced by the oracle's own pairs."""
    w = W5
    mode = layer % 3
    sh = LayerShape(w.T, w.H, w.W, NH, w.head_dim, mode, *w.boxes[mode], "bf16")
    L = VMoBALayer(sh)
    qd = to_device(q, "bf16")
    L.select(qd, to_device(k, "bf16"), to_device(v, "bf16"), tau)
    torch.cuda.synchronize()
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    bits = L.sel.cpu().numpy().copy()
    g = unpack_bits(bits, L.n_blocks)
    for h in HEADS:
        S_h = O.block_scores(q[:, h:h + 1], B[h:h + 1], SCALE)[0]
        m, st = O.threshold_select(S_h, tau)
        assert pair_set_mismatch(g[h], S_h, m, st["cut_score"]) == 0
        # density bound of the pages' stopping rule: k / (s N_b) < tau + 1 / (s N_b)
        assert st["k"] < tau * m.size + 1
        bits[h] = pack_bits(m)
        g[h] = m
    L.use_selection(torch.from_numpy(bits).cuda())
    return L, qd, g, blk


@pytest.mark.parametrize("layer", [0, 1, 2])
@pytest.mark.parametrize("tau", W5.taus)
def test_stack_selection_and_forward(layer, tau):
    q, k, v = _layer_inputs(layer)
    L, qd, g, blk = _select_and_pin(layer, tau, q, k, v)
    out, lse = L.forward(qd)
    torch.cuda.synchronize()
    got, lg = from_device(out), from_device(lse)
    for h in HEADS:
        empty = np.flatnonzero(~g[h].any(axis=1))[:8]
        rows = sample_rows(W5.s, 96, seed=1000 * layer + h, must=empty)
        o_ref, l_ref = O.attention_fwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, SCALE, rows)
        assert out_err(got[rows, h], o_ref, "bf16") <= TOL["bf16"]
        fin = np.isfinite(l_ref)
        assert np.array_equal(np.isfinite(lg[h, rows]), fin)
        if fin.any():
            assert np.abs(lg[h, rows][fin] - l_ref[fin]).max() <= 1e-3


@pytest.mark.parametrize("layer", [3, 4, 5])
def test_stack_backward(layer):
    q, k, v, dout = _layer_inputs(layer, with_dout=True)
    L, qd, g, blk = _select_and_pin(layer, 0.25, q, k, v)
    L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, "bf16"))
    torch.cuda.synchronize()
    gq, gk, gv = from_device(dq), from_device(dk), from_device(dv)
    for h in HEADS:
        empty = np.flatnonzero(~g[h].any(axis=1))[:8]
        rows = sample_rows(W5.s, 64, seed=2000 * layer + h, must=empty)
        dq_ref, _, _ = O.attention_bwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, SCALE, rows,
                                            dout[rows, h])
        assert out_err(gq[rows, h], dq_ref, "bf16") <= TOL["bf16"]
        counts = g[h].sum(axis=0)
        for j in np.flatnonzero(counts == 0):
            keys = np.flatnonzero(blk == j)
            assert np.all(gk[keys, h] == 0) and np.all(gv[keys, h] == 0)
        # every key of the most- and the least-selected block (only their
        # selecting queries reach them)
        order = [j for j in np.argsort(counts, kind="stable") if counts[j] > 0]
        for j in (int(np.argmax(counts)), order[0]):
            keys, dk_ref, dv_ref = O.attention_bwd_block_keys(q[:, h], k[:, h], v[:, h], g[h],
                                                              blk, SCALE, dout[:, h], j)
            assert out_err(gk[keys, h], dk_ref, "bf16") <= TOL["bf16"]
            assert out_err(gv[keys, h], dv_ref, "bf16") <= TOL["bf16"]


def test_stack_pair_sets_all_30_layers():
    """Every layer of the 30-layer stack at tau 0.25 (mode = layer mod 3,
    per-head gains): the GPU pair set of two heads equals the oracle's outside
    the 1e-4 band around each head's cut.  The oracle runs in spawned worker
    processes while the GPU selects."""
    import multiprocessing as mp
    w = W5
    tau = 0.25
    heads = (0, 1)
    ctx = mp.get_context("spawn")
    n_layers = w.layers
    with ctx.Pool(min(8, n_layers)) as pool:
        jobs = pool.starmap_async(oracle_jobs.stack_layer_selection,
                                  [(l, tau, heads) for l in range(n_layers)], chunksize=1)
        results = jobs.get(timeout=1800)
    for layer, q, k, masks, bands, ks in results:
        mode = layer % 3
        sh = LayerShape(w.T, w.H, w.W, len(heads), w.head_dim, mode, *w.boxes[mode], "bf16")
        L = VMoBALayer(sh)
        kd = to_device(k.astype(np.float64), "bf16")
        L.select(to_device(q.astype(np.float64), "bf16"), kd, kd, tau)
        torch.cuda.synchronize()
        g = unpack_bits(L.sel.cpu().numpy(), L.n_blocks)
        st = L.head_stats()
        for i in range(len(heads)):
            n = g[i].size
            m = np.unpackbits(masks[i], count=n).astype(bool).reshape(g[i].shape)
            band = np.unpackbits(bands[i], count=n).astype(bool).reshape(g[i].shape)
            assert int(((g[i] != m) & ~band).sum()) == 0, (layer, i)
            assert ks[i] < tau * n + 1
            assert abs(int(st["n_selected"][i]) - ks[i]) <= int(band.sum())
        del L
