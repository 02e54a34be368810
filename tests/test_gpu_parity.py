"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small workloads (256 and 2048 tokens) are compared in full: partition copies
bit-exact, block means, the selected pair set (bit-exact outside the 1e-4
relative band around each head's cut score), and O/LSE/dQ/dK/dV within the
max-abs tolerance of the I/O dtype.  Attention parity feeds the oracle's own
selection bitmap to the kernels (the ABI accepts any bitmap), so the two
sides attend to exactly the same pairs.
"""
import numpy as np
import pytest

import oracle as O
from synth import WORKLOADS

from .gpu_util import (TOL, default_scale, from_device, out_err, pack_bits,
                       pair_set_mismatch, to_device, unpack_bits, workload_arrays)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU runs select -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape  # noqa: E402
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402


def _shape(w, mode):
    bt, bh, bw = w.boxes[mode]
    return LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, mode, bt, bh, bw, w.dtype)


def _oracle_select(q, k, w, mode, tau):
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    S = O.block_scores(q, B, default_scale(w.head_dim))
    sel, stats = O.select_all_heads(S, tau)
    return box, B, S, sel, stats


CASES_SMALL = [(1, m, 0.5) for m in range(3)] + \
              [(2, m, t) for m in range(3) for t in (0.25, 0.5, 0.75)]


@pytest.mark.parametrize("wid,mode", [(1, 0), (1, 1), (1, 2), (2, 0), (2, 1), (2, 2)])
def test_partition_and_pool(wid, mode):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    sh = _shape(w, mode)
    L = VMoBALayer(sh)
    L.partition_only(to_device(k, w.dtype), to_device(v, w.dtype))
    torch.cuda.synchronize()
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    perm = O.partition_order(w.T, w.H, w.W, box)
    np.testing.assert_array_equal(from_device(L.k_perm), O.permute_keys(k, perm))
    np.testing.assert_array_equal(from_device(L.v_perm), O.permute_keys(v, perm))
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    np.testing.assert_allclose(from_device(L.blocks), B, rtol=2e-7, atol=1e-7)


@pytest.mark.parametrize("wid,mode,tau", CASES_SMALL)
def test_selection_pair_set(wid, mode, tau):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    sh = _shape(w, mode)
    L = VMoBALayer(sh)
    L.select(to_device(q, w.dtype), to_device(k, w.dtype), to_device(v, w.dtype), tau)
    torch.cuda.synchronize()
    box, B, S, sel, stats = _oracle_select(q, k, w, mode, tau)
    g = unpack_bits(L.sel.cpu().numpy(), B.shape[1])
    st = L.head_stats()
    for h in range(w.n_heads):
        assert pair_set_mismatch(g[h], S[h], sel[h], stats[h]["cut_score"]) == 0
        band = np.abs(S[h] - stats[h]["cut_score"]) <= 1e-4 * abs(stats[h]["cut_score"])
        assert abs(int(st["n_selected"][h]) - stats[h]["k"]) <= band.sum()
        assert int(st["n_selected"][h]) == int(g[h].sum())
        assert abs(st["mass"][h] - stats[h]["mass"]) < 1e-4
        assert st["mass"][h] >= tau - 1e-6 or st["all_selected"][h]


@pytest.mark.parametrize("wid,mode,tau", CASES_SMALL)
def test_attention_forward(wid, mode, tau):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    sh = _shape(w, mode)
    box, B, S, sel, _ = _oracle_select(q, k, w, mode, tau)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    scale = default_scale(w.head_dim)
    Oref, lse_ref = O.attention_fwd(q, k, v, sel, blk, scale)
    L = VMoBALayer(sh)
    qd = to_device(q, w.dtype)
    L.partition_only(to_device(k, w.dtype), to_device(v, w.dtype))
    L.use_selection(torch.from_numpy(pack_bits(sel)).cuda())
    out, lse = L.forward(qd)
    torch.cuda.synchronize()
    err = out_err(from_device(out), Oref, w.dtype)
    assert err <= TOL[w.dtype], err
    lg = from_device(lse)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lg), fin)
    assert np.abs(lg[fin] - lse_ref[fin]).max() <= 1e-3
    assert np.all(from_device(out).transpose(1, 0, 2)[~fin] == 0)


@pytest.mark.parametrize("mode,tau", [(m, t) for m in range(3) for t in (0.25, 0.5, 0.75)])
def test_attention_backward(mode, tau):
    w = WORKLOADS[2]
    q, k, v, dout = workload_arrays(w, mode, with_dout=True)
    sh = _shape(w, mode)
    box, B, S, sel, _ = _oracle_select(q, k, w, mode, tau)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    scale = default_scale(w.head_dim)
    dQ, dK, dV = O.attention_bwd(q, k, v, sel, blk, scale, dout)
    L = VMoBALayer(sh)
    qd = to_device(q, w.dtype)
    L.partition_only(to_device(k, w.dtype), to_device(v, w.dtype))
    L.use_selection(torch.from_numpy(pack_bits(sel)).cuda())
    L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, w.dtype))
    torch.cuda.synchronize()
    for name, got, ref in (("dq", dq, dQ), ("dk", dk, dK), ("dv", dv, dV)):
        err = out_err(from_device(got), ref, w.dtype)
        assert err <= TOL[w.dtype], (name, err)


def test_fp32_backward_tiny():
    w = WORKLOADS[1]
    from synth.video_latents import make_dout, round_to
    q, k, v = workload_arrays(w, 2)
    dout = round_to(make_dout(w.wid, 2, w.s, w.n_heads, w.head_dim), "f32")
    sh = _shape(w, 2)
    box, B, S, sel, _ = _oracle_select(q, k, w, 2, 0.5)
    blk = O.block_of_token(w.T, w.H, w.W, box)
    dQ, dK, dV = O.attention_bwd(q, k, v, sel, blk, default_scale(w.head_dim), dout)
    L = VMoBALayer(sh)
    qd = to_device(q, "f32")
    L.partition_only(to_device(k, "f32"), to_device(v, "f32"))
    L.use_selection(torch.from_numpy(pack_bits(sel)).cuda())
    L.forward(qd)
    dq, dk, dv = L.backward(qd, to_device(dout, "f32"))
    torch.cuda.synchronize()
    for got, ref in ((dq, dQ), (dk, dK), (dv, dV)):
        assert out_err(from_device(got), ref, "f32") <= 1e-4


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_layer_chain_on_gpu_selection(mode):
    """Partition -> select -> attention all on the GPU; rows whose selection
    equals the oracle's must match the oracle's output."""
    w = WORKLOADS[2]
    tau = 0.5
    q, k, v = workload_arrays(w, mode)
    sh = _shape(w, mode)
    L = VMoBALayer(sh)
    L.step(to_device(q, w.dtype), to_device(k, w.dtype), to_device(v, w.dtype), tau)
    torch.cuda.synchronize()
    box, B, S, sel, _ = _oracle_select(q, k, w, mode, tau)
    g = unpack_bits(L.sel.cpu().numpy(), B.shape[1])
    same = np.all(g == sel, axis=2)                       # [n_h][s]
    assert same.mean() > 0.99
    blk = O.block_of_token(w.T, w.H, w.W, box)
    Oref, _ = O.attention_fwd(q, k, v, sel, blk, default_scale(w.head_dim))
    got = from_device(L.out)
    for h in range(w.n_heads):
        rows = np.flatnonzero(same[h])
        assert out_err(got[rows, h], Oref[rows, h], w.dtype) <= TOL[w.dtype]


# ------------------------------------------------------------ edge cases

def _custom(wid, mode, q, k, v, tau):
    w = WORKLOADS[wid]
    sh = _shape(w, mode)
    L = VMoBALayer(sh)
    L.step(to_device(q, w.dtype), to_device(k, w.dtype), to_device(v, w.dtype), tau)
    torch.cuda.synchronize()
    return L


@pytest.mark.parametrize("wid", [1, 2])
def test_exact_ties_follow_index_order(wid):
    """All scores equal (K = 0): the kept pairs are the first k* in (query, block) order."""
    w = WORKLOADS[wid]
    q, _, v = workload_arrays(w, 2)
    k = np.zeros_like(q)
    tau = 0.3
    L = _custom(wid, 2, q, k, v, tau)
    box, B, S, sel, stats = _oracle_select(q, k, w, 2, tau)
    g = unpack_bits(L.sel.cpu().numpy(), B.shape[1])
    np.testing.assert_array_equal(g, sel)


def test_full_threshold_is_dense_attention():
    w = WORKLOADS[1]
    q, k, v = workload_arrays(w, 1)
    L = _custom(1, 1, q, k, v, 1.0)
    assert L.sel.cpu().numpy().view(np.uint32).min() > 0
    assert L.head_stats()["all_selected"].all()
    g = unpack_bits(L.sel.cpu().numpy(), L.n_blocks)
    assert g.all()
    out, _ = L.forward(to_device(q, w.dtype))
    torch.cuda.synchronize()
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0].permute(1, 0, 2).numpy()
    assert out_err(from_device(out), ref, "f32") <= 1e-4


def test_tiny_tau_keeps_one_pair_and_empty_rows_are_zero():
    w = WORKLOADS[2]
    q, k, v, dout = workload_arrays(w, 2, with_dout=True)
    L = _custom(2, 2, q, k, v, 1e-7)
    st = L.head_stats()
    assert np.all(st["n_selected"] == 1)
    out, lse = L.forward(to_device(q, w.dtype))
    dq, dk, dv = L.backward(to_device(q, w.dtype), to_device(dout, w.dtype))
    torch.cuda.synchronize()
    g = unpack_bits(L.sel.cpu().numpy(), L.n_blocks)
    rows_on = g.any(axis=2)                                # [n_h][s]
    o = from_device(out).transpose(1, 0, 2)
    assert np.all(o[~rows_on] == 0)
    assert np.all(np.isneginf(from_device(lse)[~rows_on]))
    assert np.all(from_device(dq).transpose(1, 0, 2)[~rows_on] == 0)
    assert np.all(np.isfinite(from_device(dk))) and np.all(np.isfinite(from_device(dv)))


def test_repeat_calls_are_deterministic():
    w = WORKLOADS[2]
    q, k, v, dout = workload_arrays(w, 0, with_dout=True)
    sh = _shape(w, 0)
    outs = []
    for _ in range(2):
        L = VMoBALayer(sh)
        L.step(to_device(q, w.dtype), to_device(k, w.dtype), to_device(v, w.dtype), 0.5,
               dout=to_device(dout, w.dtype))
        torch.cuda.synchronize()
        outs.append([x.clone() for x in (L.sel, L.out, L.lse, L.dq, L.dk, L.dv)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
