"""The ablation's selection variants on the GPU against the fp64 oracle.

Pair sets are compared bit for bit outside the 1e-4 relative band around
each cut score (the head's cut for the global rules, each row's own cut for
the local ones); pair counts of the top-k rules are integers and must match
exactly.  The small workloads are compared in full for every mode; the
55296-token layers on two heads; and the training-free setting (3D blocks,
local top-k) is run through the attention forward.
"""
import math

import numpy as np
import pytest

import oracle as O
import synth
from synth import WORKLOADS
from synth.video_latents import round_to

from .gpu_util import (BAND_REL, TOL, default_scale, from_device, out_err, pack_bits,
                       pair_set_mismatch, sample_rows, to_device, unpack_bits, workload_arrays)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

from block_sparse_attention_layer_b200 import LayerShape, decode_stats  # noqa: E402
from block_sparse_attention_layer_b200.layer import VMoBALayer  # noqa: E402


def _row_mismatch(g, S, m, cuts):
    band = np.abs(S - cuts[:, None]) <= BAND_REL * np.abs(cuts)[:, None]
    return int(((g != m) & ~band).sum())


def _run(w, mode, q, k, v, variant, param, heads=None):
    nh = w.n_heads if heads is None else heads
    sh = LayerShape(w.T, w.H, w.W, nh, w.head_dim, mode, *w.boxes[mode], w.dtype)
    L = VMoBALayer(sh)
    L.select_variant(to_device(q, w.dtype), to_device(k, w.dtype), to_device(v, w.dtype),
                     variant, param)
    torch.cuda.synchronize()
    g = unpack_bits(L.sel.cpu().numpy(), L.n_blocks)
    return L, g, decode_stats(L.stats)


def _scores(w, mode, q, k):
    box = O.mode_box(mode, w.T, w.H, w.W, *w.boxes[mode])
    B = O.pool_blocks(k, w.T, w.H, w.W, box)
    return O.block_scores(q, B, default_scale(w.head_dim))


SMALL = [(1, m) for m in range(3)] + [(2, m) for m in range(3)]


@pytest.mark.parametrize("wid,mode", SMALL)
def test_topk_global_small(wid, mode):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    S = _scores(w, mode, q, k)
    pool = S.shape[1] * S.shape[2]
    k_star = O.threshold_select(S[0], 0.25)[1]["k"]
    for kk in (1, 37, k_star, pool, pool + 5):
        _, g, st = _run(w, mode, q, k, v, "topk_global", kk)
        for h in range(w.n_heads):
            m, so = O.topk_global_select(S[h], kk)
            assert int(st["n_selected"][h]) == min(kk, pool) == g[h].sum()
            assert pair_set_mismatch(g[h], S[h], m, so["cut_score"]) == 0
            assert math.isclose(st["mass"][h], so["mass"], rel_tol=1e-4, abs_tol=1e-9)
            assert bool(st["all_selected"][h]) == (kk >= pool)


@pytest.mark.parametrize("wid,mode", SMALL)
def test_threshold_local_small(wid, mode):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    S = _scores(w, mode, q, k)
    for tau in (0.1, 0.5, 0.9, 1.0):
        _, g, st = _run(w, mode, q, k, v, "threshold_local", tau)
        for h in range(w.n_heads):
            m, so = O.threshold_local_select(S[h], tau)
            assert _row_mismatch(g[h], S[h], m, so["cut_scores"]) == 0
            assert np.all(g[h].sum(axis=1) >= 1)
            assert math.isclose(st["mass"][h], so["mass"], rel_tol=1e-4)
            assert math.isnan(st["cut_score"][h])


@pytest.mark.parametrize("wid,mode", SMALL)
def test_topk_local_small(wid, mode):
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    S = _scores(w, mode, q, k)
    nb = S.shape[2]
    for kk in (1, 3, nb, nb + 2):
        _, g, st = _run(w, mode, q, k, v, "topk_local", kk)
        for h in range(w.n_heads):
            m, so = O.topk_local_select(S[h], kk)
            assert np.all(g[h].sum(axis=1) == min(kk, nb))
            assert int(st["n_selected"][h]) == min(kk, nb) * w.s
            assert _row_mismatch(g[h], S[h], m, so["cut_scores"]) == 0
            assert math.isclose(st["mass"][h], so["mass"], rel_tol=1e-4)


def test_threshold_global_variant_is_the_method():
    w = WORKLOADS[2]
    q, k, v = workload_arrays(w, 2)
    _, g, st = _run(w, 2, q, k, v, "threshold_global", 0.25)
    sh = LayerShape(w.T, w.H, w.W, w.n_heads, w.head_dim, 2, *w.boxes[2], w.dtype)
    L = VMoBALayer(sh)
    L.select(to_device(q, w.dtype), to_device(k, w.dtype), to_device(v, w.dtype), 0.25)
    torch.cuda.synchronize()
    assert np.array_equal(unpack_bits(L.sel.cpu().numpy(), L.n_blocks), g)
    assert np.array_equal(decode_stats(L.stats)["n_selected"], st["n_selected"])


@pytest.mark.parametrize("variant,param", [("topk_global", 400000), ("threshold_local", 0.25),
                                           ("topk_local", 12)])
def test_variants_full_size_3d(variant, param):
    """55296-token 3D layer (288 blocks), two heads."""
    w = WORKLOADS[4]
    nh = 2
    q, k, v = synth.make_qkv(w.wid, 30, w.T, w.H, w.W, nh, w.head_dim)
    q, k, v = (round_to(x, "bf16") for x in (q, k, v))
    _, g, st = _run(w, 2, q, k, v, variant, param, heads=nh)
    S = _scores(w, 2, q, k)
    for h in range(nh):
        if variant == "topk_global":
            m, so = O.topk_global_select(S[h], param)
            assert int(st["n_selected"][h]) == param
            assert pair_set_mismatch(g[h], S[h], m, so["cut_score"]) == 0
        elif variant == "threshold_local":
            m, so = O.threshold_local_select(S[h], param)
            assert _row_mismatch(g[h], S[h], m, so["cut_scores"]) == 0
        else:
            m, so = O.topk_local_select(S[h], param)
            assert np.all(g[h].sum(axis=1) == param)
            assert _row_mismatch(g[h], S[h], m, so["cut_scores"]) == 0


def test_training_free_setting_attention():
    """3D blocks with local top-k (digest App. A: the training-free runs),
    then the attention forward on the oracle's own pairs, sampled rows."""
    w = WORKLOADS[4]
    nh = 2
    kk = 8
    scale = 1 / math.sqrt(128)
    q, k, v = synth.make_qkv(w.wid, 31, w.T, w.H, w.W, nh, w.head_dim)
    q, k, v = (round_to(x, "bf16") for x in (q, k, v))
    L, g, _ = _run(w, 2, q, k, v, "topk_local", kk, heads=nh)
    S = _scores(w, 2, q, k)
    box = O.mode_box(2, w.T, w.H, w.W, *w.boxes[2])
    blk = O.block_of_token(w.T, w.H, w.W, box)
    bits = L.sel.cpu().numpy().copy()
    for h in range(nh):
        m, so = O.topk_local_select(S[h], kk)
        assert _row_mismatch(g[h], S[h], m, so["cut_scores"]) == 0
        bits[h] = pack_bits(m)
        g[h] = m
    L.use_selection(torch.from_numpy(bits).cuda())
    out, _ = L.forward(to_device(q, "bf16"))
    torch.cuda.synchronize()
    got = from_device(out)
    for h in range(nh):
        rows = sample_rows(w.s, 128, seed=700 + h)
        o_ref, _ = O.attention_fwd_rows(q[:, h], k[:, h], v[:, h], g[h], blk, scale, rows)
        assert out_err(got[rows, h], o_ref, "bf16") <= TOL["bf16"]


def _rownorm_logp(S_h):
    m = S_h.max(axis=1, keepdims=True)
    return S_h - (m + np.log(np.exp(S_h - m).sum(axis=1, keepdims=True)))


@pytest.mark.parametrize("wid,mode", SMALL)
@pytest.mark.parametrize("tau", [0.25, 0.6])
def test_rownorm_global_small(wid, mode, tau):
    """The per-query reading of the normalisation as a selection variant: the
    pair set equals the oracle's outside the 1e-4 band around the cut in its
    own ranking value (the log row softmax); k and the mass match."""
    w = WORKLOADS[wid]
    q, k, v = workload_arrays(w, mode)
    L, g, st = _run(w, mode, q, k, v, "rownorm_global", tau)
    S = _scores(w, mode, q, k)
    for h in range(w.n_heads):
        m, ost = O.rownorm_global_select(S[h], tau)
        lp = _rownorm_logp(S[h])
        assert pair_set_mismatch(g[h], lp, m, ost["cut_logp"]) == 0
        band = np.abs(lp - ost["cut_logp"]) <= BAND_REL * abs(ost["cut_logp"])
        assert abs(int(st["n_selected"][h]) - ost["k"]) <= int(band.sum())
        assert abs(float(st["mass"][h]) - ost["mass"]) < 1e-4
        assert abs(float(st["cut_score"][h]) - ost["cut_logp"]) <= 1e-4 * abs(ost["cut_logp"]) \
            + 1e-5


@pytest.mark.parametrize("mode", [0, 2])
def test_rownorm_global_full_size(mode):
    w = WORKLOADS[4]
    nh = 2
    q, k, v = synth.make_qkv(w.wid, 30 + mode, w.T, w.H, w.W, nh, w.head_dim)
    q, k, v = (round_to(x, "bf16") for x in (q, k, v))
    L, g, st = _run(w, mode, q, k, v, "rownorm_global", 0.25, heads=nh)
    S = _scores(w, mode, q, k)
    for h in range(nh):
        m, ost = O.rownorm_global_select(S[h], 0.25)
        lp = _rownorm_logp(S[h])
        assert pair_set_mismatch(g[h], lp, m, ost["cut_logp"]) == 0
