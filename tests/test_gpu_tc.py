"""Tensor-core path (bf16, head_dim 128) against the fp64 oracle.

Small shapes are compared on every output element; the 32760- and 55296-token
layers (ragged 60-token blocks; the headline shape) are compared on sampled
query rows of two heads, with those heads attending the oracle's own
selection, plus the full pair set of those heads.
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from synth.video_latents import round_to

from .gpu_util import (TOL, from_device, out_err, pack_bits, pair_set_mismatch, sample_rows,
                       to_device, unpack_bits)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape  # noqa: E402
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402

# (name, T, H, W, heads, boxes per mode)
SMALL = [
    ("2048tok", 8, 16, 16, 2, ((1, 16, 16), (8, 4, 4), (2, 4, 4))),
    ("360tok-ragged", 3, 10, 12, 2, ((1, 10, 12), (3, 5, 4), (1, 5, 4))),
]


def _inputs(seed, T, H, W, nh, with_dout=False):
    q, k, v = synth.make_qkv(100 + seed, 0, T, H, W, nh, 128)
    out = [round_to(x, "bf16") for x in (q, k, v)]
    if with_dout:
        out.append(round_to(synth.make_dout(100 + seed, 0, T * H * W, nh, 128), "bf16"))
    return out


def _oracle_sel(q, k, T, H, W, mode, box_cfg, tau):
    box = O.mode_box(mode, T, H, W, *box_cfg)
    S = O.block_scores(q, O.pool_blocks(k, T, H, W, box), 1 / math.sqrt(128))
    sel, stats = O.select_all_heads(S, tau)
    return box, S, sel, stats


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("tau", [0.25, 0.6, 1.0])
def test_tc_forward_small(case, mode, tau):
    name, T, H, W, nh, boxes = SMALL[case]
    q, k, v = _inputs(case, T, H, W, nh)
    box, S, sel, _ = _oracle_sel(q, k, T, H, W, mode, boxes[mode], tau)
    blk = O.block_of_token(T, H, W, box)
    Oref, lse_ref = O.attention_fwd(q, k, v, sel, blk, 1 / math.sqrt(128))
    sh = LayerShape(T, H, W, nh, 128, mode, *boxes[mode], "bf16")
    L = VMoBALayer(sh)
    L.partition_only(to_device(k, "bf16"), to_device(v, "bf16"))
    L.use_selection(torch.from_numpy(pack_bits(sel)).cuda())
    out, lse = L.forward(to_device(q, "bf16"))
    torch.cuda.synchronize()
    assert out_err(from_device(out), Oref, "bf16") <= TOL["bf16"]
    lg = from_device(lse)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lg), fin)
    if fin.any():
        assert np.abs(lg[fin] - lse_ref[fin]).max() <= 1e-3


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("mode", [0, 2])
def test_backward_after_tc_forward(case, mode):
    name, T, H, W, nh, boxes = SMALL[case]
    q, k, v, dout = _inputs(case, T, H, W, nh, with_dout=True)
    tau = 0.4
    box, S, sel, _ = _oracle_sel(q, k, T, H, W, mode, boxes[mode], tau)
    blk = O.block_of_token(T, H, W, box)
    dQ, dK, dV = O.attention_bwd(q, k, v, sel, blk, 1 / math.sqrt(128), dout)
    sh = LayerShape(T, H, W, nh, 128, mode, *boxes[mode], "bf16")
    L = VMoBALayer(sh)
    qd = to_device(q, "bf16")
    L.partition_only(to_device(k, "bf16"), to_device(v, "bf16"))
    L.use_selection(torch.from_numpy(pack_bits(sel)).cuda())
    L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, "bf16"))
    torch.cuda.synchronize()
    for name_, got, ref in (("dq", dq, dQ), ("dk", dk, dK), ("dv", dv, dV)):
        assert out_err(from_device(got), ref, "bf16") <= TOL["bf16"], name_


def test_tc_forward_empty_rows_and_single_pair():
    name, T, H, W, nh, boxes = SMALL[0]
    q, k, v = _inputs(7, T, H, W, nh)
    sh = LayerShape(T, H, W, nh, 128, 2, *boxes[2], "bf16")
    L = VMoBALayer(sh)
    L.step(to_device(q, "bf16"), to_device(k, "bf16"), to_device(v, "bf16"), 1e-7)
    torch.cuda.synchronize()
    assert np.all(L.head_stats()["n_selected"] == 1)
    g = unpack_bits(L.sel.cpu().numpy(), L.n_blocks)
    rows_on = g.any(axis=2)
    o = from_device(L.out).transpose(1, 0, 2)
    assert np.all(o[~rows_on] == 0)
    assert np.all(np.isneginf(from_device(L.lse)[~rows_on]))
    box = O.mode_box(2, T, H, W, *boxes[2])
    Oref, _ = O.attention_fwd(q, k, v, g, O.block_of_token(T, H, W, box), 1 / math.sqrt(128))
    assert out_err(from_device(L.out), Oref, "bf16") <= TOL["bf16"]


@pytest.mark.parametrize("wid,mode", [(3, 0), (3, 1), (3, 2), (4, 0), (4, 1), (4, 2)])
def test_tc_forward_full_size_sampled(wid, mode):
    w = synth.WORKLOADS[wid]
    heads = (0, w.n_heads // 3, 2 * w.n_heads // 3, w.n_heads - 1)
    tau = 0.25
    q, k, v = synth.make_qkv(w.wid, mode, w.T, w.H, w.W, w.n_heads, w.head_dim)
    q, k, v = (round_to(x, "bf16") for x in (q, k, v))
    sh = LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, mode, *w.boxes[mode], "bf16")
    L = VMoBALayer(sh)
    qd = to_device(q, "bf16")
    L.select(qd, to_device(k, "bf16"), to_device(v, "bf16"), tau)
    torch.cuda.synchronize()
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    bits = L.sel.cpu().numpy().copy()
    g = unpack_bits(bits, L.n_blocks)
    for h in heads:
        S_h = O.block_scores(q[:, h:h + 1], B[h:h + 1], 1 / math.sqrt(128))[0]
        m, st = O.threshold_select(S_h, tau)
        assert pair_set_mismatch(g[h], S_h, m, st["cut_score"]) == 0
        bits[h] = pack_bits(m)          # attend the oracle's own pairs on checked heads
        g[h] = m
    L.use_selection(torch.from_numpy(bits).cuda())
    out, lse = L.forward(qd)
    torch.cuda.synchronize()
    got = from_device(out)
    lg = from_device(lse)
    for h in heads:
        empty = np.flatnonzero(~g[h].any(axis=1))[:8]
        rows = sample_rows(w.s, 192, seed=h, must=empty)
        o_ref, l_ref = O.attention_fwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk,
                                            1 / math.sqrt(128), rows)
        assert out_err(got[rows, h], o_ref, "bf16") <= TOL["bf16"]
        fin = np.isfinite(l_ref)
        assert np.array_equal(np.isfinite(lg[h, rows]), fin)
        if fin.any():
            assert np.abs(lg[h, rows][fin] - l_ref[fin]).max() <= 1e-3


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_tc_backward_full_size(mode):
    """55296-token layer, fwd + bwd on the tensor cores.  Two heads attend the
    oracle's own pairs; dQ is compared on sampled rows; dK/dV on every key of
    the block with the MOST selecting queries (thousands: hundreds of query
    tiles accumulate in the key-stationary pass, the longest list launched
    first) and of the block with the fewest, and keys of blocks nobody
    selected must get exact zeros."""
    w = synth.WORKLOADS[4]
    heads = (0, w.n_heads - 1)
    tau = 0.25
    scale = 1 / math.sqrt(128)
    q, k, v = synth.make_qkv(w.wid, 10 + mode, w.T, w.H, w.W, w.n_heads, w.head_dim)
    dout = synth.make_dout(w.wid, 10 + mode, w.s, w.n_heads, w.head_dim)
    q, k, v, dout = (round_to(x, "bf16") for x in (q, k, v, dout))
    sh = LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, mode, *w.boxes[mode], "bf16")
    L = VMoBALayer(sh)
    qd = to_device(q, "bf16")
    L.select(qd, to_device(k, "bf16"), to_device(v, "bf16"), tau)
    torch.cuda.synchronize()
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    bits = L.sel.cpu().numpy().copy()
    g = unpack_bits(bits, L.n_blocks)
    for h in heads:
        S_h = O.block_scores(q[:, h:h + 1], B[h:h + 1], scale)[0]
        m, _ = O.threshold_select(S_h, tau)
        bits[h] = pack_bits(m)
        g[h] = m
    L.use_selection(torch.from_numpy(bits).cuda())
    L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, "bf16"))
    torch.cuda.synchronize()
    gq, gk, gv = from_device(dq), from_device(dk), from_device(dv)
    for h in heads:
        empty = np.flatnonzero(~g[h].any(axis=1))[:8]
        rows = sample_rows(w.s, 128, seed=100 + h, must=empty)
        dq_ref, _, _ = O.attention_bwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, scale, rows,
                                            dout[rows, h])
        assert out_err(gq[rows, h], dq_ref, "bf16") <= TOL["bf16"]
        counts = g[h].sum(axis=0)
        for j in np.flatnonzero(counts == 0):
            keys = np.flatnonzero(blk == j)
            assert np.all(gk[keys, h] == 0) and np.all(gv[keys, h] == 0)
        order = [j for j in np.argsort(counts, kind="stable") if counts[j] > 0]
        most = int(np.argmax(counts))
        assert counts[most] > 8 * 128          # a long query list
        for j in (most, order[0]):
            keys, dk_ref, dv_ref = O.attention_bwd_block_keys(q[:, h], k[:, h], v[:, h], g[h],
                                                              blk, scale, dout[:, h], j)
            assert out_err(gk[keys, h], dk_ref, "bf16") <= TOL["bf16"]
            assert out_err(gv[keys, h], dv_ref, "bf16") <= TOL["bf16"]


@pytest.mark.parametrize("mode", [0, 2])
def test_paper_block_counts_fwd_bwd(mode):
    """The paper's 8-48-72 block counts on the 55296-token latent (1D: 3-frame
    blocks of 6912 keys; 3D: 4x12x16 boxes of 768 keys; 2D is workload 4's):
    full pair sets of two heads, then forward rows and dQ rows on the oracle's
    pairs, and every key of the least-selected block."""
    w = synth.WORKLOADS[4]
    box_cfg = synth.BOXES_8_48_72[mode]
    nh = 2
    tau = 0.25
    scale = 1 / math.sqrt(128)
    q, k, v = synth.make_qkv(w.wid, 20 + mode, w.T, w.H, w.W, nh, w.head_dim)
    dout = synth.make_dout(w.wid, 20 + mode, w.s, nh, w.head_dim)
    q, k, v, dout = (round_to(x, "bf16") for x in (q, k, v, dout))
    sh = LayerShape(w.T, w.H, w.W, nh, w.head_dim, mode, *box_cfg, "bf16")
    L = VMoBALayer(sh)
    qd = to_device(q, "bf16")
    L.select(qd, to_device(k, "bf16"), to_device(v, "bf16"), tau)
    torch.cuda.synchronize()
    box = O.mode_box(mode, w.T, w.H, w.W, *box_cfg)
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    bits = L.sel.cpu().numpy().copy()
    g = unpack_bits(bits, L.n_blocks)
    for h in range(nh):
        S_h = O.block_scores(q[:, h:h + 1], B[h:h + 1], scale)[0]
        m, st = O.threshold_select(S_h, tau)
        assert pair_set_mismatch(g[h], S_h, m, st["cut_score"]) == 0
        bits[h] = pack_bits(m)
        g[h] = m
    L.use_selection(torch.from_numpy(bits).cuda())
    out, _ = L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, "bf16"))
    torch.cuda.synchronize()
    go, gq, gk, gv = from_device(out), from_device(dq), from_device(dk), from_device(dv)
    for h in range(nh):
        empty = np.flatnonzero(~g[h].any(axis=1))[:8]
        rows = sample_rows(w.s, 96, seed=300 + h, must=empty)
        o_ref, _ = O.attention_fwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, scale, rows)
        assert out_err(go[rows, h], o_ref, "bf16") <= TOL["bf16"]
        dq_ref, _, _ = O.attention_bwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, scale, rows,
                                            dout[rows, h])
        assert out_err(gq[rows, h], dq_ref, "bf16") <= TOL["bf16"]
        counts = g[h].sum(axis=0)
        order = [j for j in np.argsort(counts, kind="stable") if counts[j] > 0]
        for j in (int(np.argmax(counts)), order[0]):
            keys, dk_ref, dv_ref = O.attention_bwd_block_keys(q[:, h], k[:, h], v[:, h], g[h],
                                                              blk, scale, dout[:, h], j)
            assert out_err(gk[keys, h], dk_ref, "bf16") <= TOL["bf16"]
            assert out_err(gv[keys, h], dv_ref, "bf16") <= TOL["bf16"]


@pytest.mark.parametrize("name", ["11520tok", "46080tok"])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_paper_10_48_60_setting(name, mode):
    """The pre-training runs' 10-48-60 block counts at 11K and 46K tokens
    (latents chosen so the counts come out exactly; see synth.workloads):
    full pair sets of two heads, then forward and dQ on sampled rows and
    dK/dV on every key of the most- and least-selected block, on the
    oracle's pairs."""
    w = synth.PAPER_10_48_60[name]
    nh, tau, scale = 2, 0.25, 1 / math.sqrt(128)
    q, k, v = synth.make_qkv(w.wid, mode, w.T, w.H, w.W, nh, w.head_dim)
    dout = synth.make_dout(w.wid, mode, w.s, nh, w.head_dim)
    q, k, v, dout = (round_to(x, "bf16") for x in (q, k, v, dout))
    sh = LayerShape(w.T, w.H, w.W, nh, w.head_dim, mode, *w.boxes[mode], "bf16")
    L = VMoBALayer(sh)
    assert L.n_blocks == (10, 48, 60)[mode]
    qd = to_device(q, "bf16")
    L.select(qd, to_device(k, "bf16"), to_device(v, "bf16"), tau)
    torch.cuda.synchronize()
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    bits = L.sel.cpu().numpy().copy()
    g = unpack_bits(bits, L.n_blocks)
    for h in range(nh):
        S_h = O.block_scores(q[:, h:h + 1], B[h:h + 1], scale)[0]
        m, st = O.threshold_select(S_h, tau)
        assert pair_set_mismatch(g[h], S_h, m, st["cut_score"]) == 0
        bits[h] = pack_bits(m)
        g[h] = m
    L.use_selection(torch.from_numpy(bits).cuda())
    out, _ = L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, "bf16"))
    torch.cuda.synchronize()
    go, gq, gk, gv = from_device(out), from_device(dq), from_device(dk), from_device(dv)
    for h in range(nh):
        empty = np.flatnonzero(~g[h].any(axis=1))[:8]
        rows = sample_rows(w.s, 96, seed=400 + h, must=empty)
        o_ref, _ = O.attention_fwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, scale, rows)
        assert out_err(go[rows, h], o_ref, "bf16") <= TOL["bf16"]
        dq_ref, _, _ = O.attention_bwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, scale, rows,
                                            dout[rows, h])
        assert out_err(gq[rows, h], dq_ref, "bf16") <= TOL["bf16"]
        counts = g[h].sum(axis=0)
        order = [j for j in np.argsort(counts, kind="stable") if counts[j] > 0]
        for j in (int(np.argmax(counts)), order[0]):
            keys, dk_ref, dv_ref = O.attention_bwd_block_keys(q[:, h], k[:, h], v[:, h], g[h],
                                                              blk, scale, dout[:, h], j)
            assert out_err(gk[keys, h], dk_ref, "bf16") <= TOL["bf16"]
            assert out_err(gv[keys, h], dv_ref, "bf16") <= TOL["bf16"]


@pytest.mark.parametrize("mode", [1, 2])
def test_selection_repeatable_on_large_pool(mode):
    """The selection's bucket masses are integer (fixed-point) sums, so two
    selections of the same 55296-token layer agree bit for bit on every head
    (the 3D pool holds 15.9 M pairs per head, where an order-dependent float
    sum moves the cut by pairs whose mass is at its rounding)."""
    from synth import torch_latents as TL
    w = synth.WORKLOADS[4]
    q, k, v = TL.make_qkv(w.wid, mode, w.T, w.H, w.W, w.n_heads, w.head_dim)
    sh = LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, mode, *w.boxes[mode], "bf16")
    L = VMoBALayer(sh, max_pair_fraction=0.25)
    runs = []
    for _ in range(3):
        L.select(q, k, v, 0.25)
        torch.cuda.synchronize()
        st = L.head_stats()
        runs.append((L.sel.cpu().numpy().copy(), st["n_selected"].copy(), st["mass"].copy()))
    for bits, n, m in runs[1:]:
        assert np.array_equal(bits, runs[0][0])
        assert np.array_equal(n, runs[0][1])
        assert np.array_equal(m, runs[0][2])
