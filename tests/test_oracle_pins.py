"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than its own formula:
a brute-force enumeration, a library routine (torch SDPA / autograd in fp64),
a closed form, an invariant stated on the pages, or a finite difference.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth


def _coords(T, H, W):
    for t in range(T):
        for y in range(H):
            for x in range(W):
                yield t, y, x


BOXES = [
    ((4, 6, 8), (1, 6, 8)),      # 1D box: whole frames
    ((4, 6, 8), (4, 3, 4)),      # 2D box: spatial patch across all frames
    ((4, 6, 8), (2, 3, 2)),      # 3D box
    ((3, 4, 5), (1, 1, 1)),      # block size 1
    ((2, 2, 2), (2, 2, 2)),      # a single block
]


# ---------------------------------------------------------------- partition

def test_mode_cycle_is_layer_mod_3():
    # notes, key design 1: l mod 3 = 0 -> 1D, = 1 -> 2D, = 2 -> 3D
    assert [O.mode_for_layer(l) for l in range(7)] == [0, 1, 2, 0, 1, 2, 0]
    assert O.mode_box(0, 4, 6, 8, 2, 3, 4) == (2, 6, 8)
    assert O.mode_box(1, 4, 6, 8, 2, 3, 4) == (4, 3, 4)
    assert O.mode_box(2, 4, 6, 8, 2, 3, 4) == (2, 3, 4)


@pytest.mark.parametrize("grid,box", BOXES)
def test_partition_matches_coordinate_enumeration(grid, box):
    T, H, W = grid
    bt, bh, bw = box
    perm = O.partition_order(T, H, W, box)
    assert sorted(perm.tolist()) == list(range(T * H * W))
    # brute force: walk blocks row-major, then (t, y, x) inside each block
    expect = []
    for pt in range(T // bt):
        for ph in range(H // bh):
            for pw in range(W // bw):
                for t in range(pt * bt, pt * bt + bt):
                    for y in range(ph * bh, ph * bh + bh):
                        for x in range(pw * bw, pw * bw + bw):
                            expect.append(t * H * W + y * W + x)
    assert perm.tolist() == expect
    blk = O.block_of_token(T, H, W, box)
    nbh, nbw = H // bh, W // bw
    for t, y, x in _coords(T, H, W):
        assert blk[t * H * W + y * W + x] == ((t // bt) * nbh + y // bh) * nbw + x // bw


def test_3d_box_spanning_an_axis_equals_1d_or_2d():
    T, H, W = 4, 6, 8
    # 3D with bt = T is the 2D partition; 3D with (bh, bw) = (H, W) is 1D
    b2 = O.mode_box(1, T, H, W, 1, 3, 4)
    b3 = O.mode_box(2, T, H, W, T, 3, 4)
    assert np.array_equal(O.partition_order(T, H, W, b2), O.partition_order(T, H, W, b3))
    b1 = O.mode_box(0, T, H, W, 2, 1, 1)
    b3 = O.mode_box(2, T, H, W, 2, H, W)
    assert np.array_equal(O.partition_order(T, H, W, b1), O.partition_order(T, H, W, b3))


def test_box_must_divide_grid():
    with pytest.raises(ValueError):
        O.partition_order(4, 6, 8, (3, 6, 8))


# --------------------------------------------------------------------- pool

@pytest.mark.parametrize("grid,box", BOXES)
def test_pool_matches_brute_force_sums(grid, box):
    T, H, W = grid
    rng = np.random.default_rng(7)
    K = rng.standard_normal((T * H * W, 2, 5))
    B = O.pool_blocks(K, T, H, W, box)
    bt, bh, bw = box
    nbh, nbw = H // bh, W // bw
    acc = np.zeros_like(B)
    cnt = np.zeros(B.shape[1])
    for t, y, x in _coords(T, H, W):
        j = ((t // bt) * nbh + y // bh) * nbw + x // bw
        acc[:, j] += K[t * H * W + y * W + x]
        cnt[j] += 1
    assert np.all(cnt == bt * bh * bw)
    np.testing.assert_allclose(B, acc / cnt[None, :, None], rtol=1e-13, atol=1e-13)
    # closed forms: the mean of the block means is the mean of all keys
    np.testing.assert_allclose(B.mean(axis=1), K.mean(axis=0), rtol=1e-12, atol=1e-13)


def test_pool_of_constant_keys_is_the_constant():
    K = np.full((4 * 6 * 8, 3, 4), 1.25)
    B = O.pool_blocks(K, 4, 6, 8, (2, 3, 2))
    assert np.all(B == 1.25)


def test_block_size_one_pool_is_the_keys():
    T, H, W = 3, 4, 5
    K = np.random.default_rng(1).standard_normal((T * H * W, 2, 4))
    B = O.pool_blocks(K, T, H, W, (1, 1, 1))
    np.testing.assert_array_equal(B, K.transpose(1, 0, 2))


# ------------------------------------------------------------------- scores

@pytest.mark.parametrize("grid,box", BOXES[:3])
def test_scores_are_block_averages_of_token_logits(grid, box):
    T, H, W = grid
    s = T * H * W
    rng = np.random.default_rng(3)
    Q = rng.standard_normal((s, 2, 8))
    K = rng.standard_normal((s, 2, 8))
    scale = 0.37
    S = O.block_scores(Q, O.pool_blocks(K, T, H, W, box), scale)
    blk = O.block_of_token(T, H, W, box)
    nb = blk.max() + 1
    for h in range(2):
        logits = scale * torch.from_numpy(Q[:, h]) @ torch.from_numpy(K[:, h]).T
        avg = np.zeros((s, nb))
        for j in range(nb):
            avg[:, j] = logits[:, torch.from_numpy(blk == j)].mean(dim=1).numpy()
        np.testing.assert_allclose(S[h], avg, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- selection

def _brute_force_min_card(p, tau):
    """Smallest subset size whose mass reaches tau, and the best mass at that size."""
    n = p.size
    for k in range(1, n + 1):
        best = max(sum(p[list(c)]) for c in itertools.combinations(range(n), k))
        if best >= tau:
            return k, best
    return n, p.sum()


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("tau", [0.1, 0.25, 0.5, 0.8])
def test_selection_brute_force_on_tiny_pools(seed, tau):
    rng = np.random.default_rng(seed)
    s, nb = (4, 3) if seed % 2 else (3, 4)
    S = rng.standard_normal((s, nb)) * (0.5 + seed)
    mask, st = O.threshold_select(S, tau)
    e = np.exp(S - S.max())
    p = (e / e.sum()).reshape(-1)
    k_bf, best = _brute_force_min_card(p, tau)
    assert st["k"] == k_bf == mask.sum()
    assert math.isclose(p[mask.reshape(-1)].sum(), best, rel_tol=1e-12)
    assert math.isclose(st["mass"], best, rel_tol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_selection_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    s, nb = 64, 12
    S = rng.standard_normal((s, nb)) * 3.0
    prev = None
    e = np.exp(S - S.max())
    p = e / e.sum()
    for tau in [0.05, 0.1, 0.25, 0.5, 0.75, 0.99]:
        mask, st = O.threshold_select(S, tau)
        k = st["k"]
        # mass reaches tau and is minimal
        assert p[mask].sum() >= tau - 1e-15
        sorted_p = np.sort(p.reshape(-1))[::-1]
        assert sorted_p[: k - 1].sum() < tau
        # density bound ("token sparsity stays below tau", notes key design 3)
        assert k / (s * nb) < tau + 1.0 / (s * nb)
        # a threshold set: every selected score >= every unselected score
        if 0 < k < s * nb:
            assert S[mask].min() >= S[~mask].max()
        assert math.isclose(st["cut_score"], S[mask].min())
        # monotone in tau (larger tau keeps more pairs)
        if prev is not None:
            assert np.all(mask[prev])
        prev = mask


def test_selection_tie_break_and_full_threshold():
    S = np.zeros((3, 2))                    # all pairs tie
    mask, st = O.threshold_select(S, 0.5)   # p = 1/6 each -> need 3 pairs
    assert st["k"] == 3
    assert mask.reshape(-1).tolist() == [True, True, True, False, False, False]
    mask, st = O.threshold_select(np.random.default_rng(0).standard_normal((5, 3)), 1.0)
    assert mask.all()
    mask, _ = O.threshold_select(np.random.default_rng(0).standard_normal((5, 3)), 2.0)
    assert mask.all()
    with pytest.raises(ValueError):
        O.threshold_select(S, 0.0)
    with pytest.raises(ValueError):
        O.threshold_select(S, float("nan"))


# -------------------------------------------- selection variants (ablation)

def _brute_best_k_subset(x, k):
    """Largest sum of any k-subset of x (enumeration)."""
    return max(sum(x[list(c)]) for c in itertools.combinations(range(x.size), k))


@pytest.mark.parametrize("seed", range(6))
def test_topk_global_brute_force_and_nesting(seed):
    rng = np.random.default_rng(300 + seed)
    S = rng.standard_normal((3, 4)) * (1 + seed)
    flat = S.reshape(-1)
    prev = None
    for k in range(1, flat.size + 1):
        mask, st = O.topk_global_select(S, k)
        m = mask.reshape(-1)
        assert m.sum() == k == st["k"]
        assert math.isclose(flat[m].sum(), _brute_best_k_subset(flat, k), rel_tol=1e-12)
        e = np.exp(S - S.max())
        assert math.isclose(st["mass"], (e / e.sum()).reshape(-1)[m].sum(), rel_tol=1e-12)
        if prev is not None:
            assert np.all(m[prev])
        prev = m
    assert O.topk_global_select(S, 10 ** 6)[0].all()


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("tau", [0.1, 0.25, 0.6])
def test_topk_global_at_k_star_is_the_threshold_rule(seed, tau):
    # the method's rule is a prefix of the same ranking: its k* pairs are the top-k*
    rng = np.random.default_rng(400 + seed)
    S = rng.standard_normal((40, 9)) * 2.0
    m_thr, st = O.threshold_select(S, tau)
    m_top, st2 = O.topk_global_select(S, st["k"])
    assert np.array_equal(m_thr, m_top)
    assert math.isclose(st["mass"], st2["mass"], rel_tol=1e-12)


def test_topk_global_ties_and_arguments():
    mask, st = O.topk_global_select(np.zeros((3, 2)), 4)     # constant pool
    assert mask.reshape(-1).tolist() == [True] * 4 + [False] * 2
    for bad in (0, -1, 1.5):
        with pytest.raises(ValueError):
            O.topk_global_select(np.zeros((2, 2)), bad)


def _brute_min_card_row(p, tau):
    for k in range(1, p.size + 1):
        best = _brute_best_k_subset(p, k)
        if best >= tau:
            return k, best
    return p.size, p.sum()


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("tau", [0.2, 0.5, 0.9])
def test_threshold_local_brute_force_per_row(seed, tau):
    rng = np.random.default_rng(500 + seed)
    S = rng.standard_normal((5, 6)) * (0.5 + seed)
    mask, st = O.threshold_local_select(S, tau)
    masses = []
    for i in range(S.shape[0]):
        e = np.exp(S[i] - S[i].max())
        p = e / e.sum()
        k_bf, best = _brute_min_card_row(p, tau)
        assert mask[i].sum() == k_bf >= 1
        assert math.isclose(p[mask[i]].sum(), best, rel_tol=1e-12)
        # minimality: without its lowest kept block the row falls short of tau
        lowest = np.flatnonzero(mask[i])[np.argmin(S[i][mask[i]])]
        assert p[mask[i]].sum() - p[lowest] < tau
        masses.append(best)
    assert st["k"] == mask.sum()
    assert math.isclose(st["mass"], float(np.mean(masses)), rel_tol=1e-12)


@pytest.mark.parametrize("tau", [0.1, 0.37, 0.8])
def test_local_rules_on_one_query_equal_global_ones(tau):
    # with a single query row the head's pool is that row: local == global
    S = np.random.default_rng(7).standard_normal((1, 11)) * 2.0
    assert np.array_equal(O.threshold_local_select(S, tau)[0], O.threshold_select(S, tau)[0])
    for k in (1, 4, 11):
        assert np.array_equal(O.topk_local_select(S, k)[0], O.topk_global_select(S, k)[0])


@pytest.mark.parametrize("seed", range(4))
def test_topk_local_brute_force_and_counts(seed):
    rng = np.random.default_rng(600 + seed)
    S = rng.standard_normal((6, 5)) * (1 + seed)
    for k in (1, 2, 4, 5, 9):
        mask, st = O.topk_local_select(S, k)
        kk = min(k, S.shape[1])
        assert np.all(mask.sum(axis=1) == kk) and st["k"] == kk * S.shape[0]
        for i in range(S.shape[0]):
            assert math.isclose(S[i][mask[i]].sum(), _brute_best_k_subset(S[i], kk),
                                rel_tol=1e-12)
    mask, _ = O.topk_local_select(np.zeros((2, 4)), 2)        # ties: lower block first
    assert mask.tolist() == [[True, True, False, False]] * 2


@pytest.mark.parametrize("tau", [0.1, 0.37, 0.8])
def test_rownorm_global_reduces_to_the_method(tau):
    rng = np.random.default_rng(11)
    # one query row: the row softmax is the pool softmax
    S = rng.standard_normal((1, 9)) * 2.0
    assert np.array_equal(O.rownorm_global_select(S, tau)[0], O.threshold_select(S, tau)[0])
    # all rows equal: p_ij = softmax(row)_j / s is the pool softmax too
    S = np.tile(rng.standard_normal(7) * 2.0, (5, 1))
    m, st = O.rownorm_global_select(S, tau)
    m_ref, st_ref = O.threshold_select(S, tau)
    assert np.array_equal(m, m_ref) and st["k"] == st_ref["k"]
    assert math.isclose(st["mass"], st_ref["mass"], rel_tol=1e-12)


def test_rownorm_global_row_shift_invariance():
    rng = np.random.default_rng(12)
    S = rng.standard_normal((6, 5)) * 1.5
    shifted = S + np.array([8.0, -3.0, 0.0, 1.5, -6.0, 2.0])[:, None]
    for tau in (0.2, 0.5, 0.9):
        assert np.array_equal(O.rownorm_global_select(S, tau)[0],
                              O.rownorm_global_select(shifted, tau)[0])
    # the method's pool softmax moves with the shift: the two readings differ
    assert not np.array_equal(O.threshold_select(S, 0.5)[0], O.threshold_select(shifted, 0.5)[0])


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("tau", [0.1, 0.25, 0.5, 0.8])
def test_rownorm_global_brute_force_on_tiny_pools(seed, tau):
    rng = np.random.default_rng(700 + seed)
    s, nb = (4, 3) if seed % 2 else (3, 4)
    S = rng.standard_normal((s, nb)) * (0.5 + seed)
    mask, st = O.rownorm_global_select(S, tau)
    e = np.exp(S - S.max(axis=1, keepdims=True))
    p = (e / e.sum(axis=1, keepdims=True) / s).reshape(-1)
    assert math.isclose(p.sum(), 1.0, rel_tol=1e-12)
    k_bf, best = _brute_force_min_card(p, tau)
    assert st["k"] == k_bf == mask.sum()
    assert math.isclose(p[mask.reshape(-1)].sum(), best, rel_tol=1e-12)
    assert math.isclose(st["mass"], best, rel_tol=1e-12)
    # minimality: without its least kept pair the mass falls short of tau
    assert best - p[mask.reshape(-1)].min() < tau
    # the cut is the last kept pair's log row softmax
    logp = np.log(p * s).reshape(S.shape)
    assert math.isclose(st["cut_logp"], logp[mask].min(), rel_tol=1e-12, abs_tol=1e-12)


def test_rownorm_global_ties_and_arguments():
    mask, st = O.rownorm_global_select(np.zeros((3, 2)), 0.5)   # p = 1/6 each
    assert st["k"] == 3
    assert mask.reshape(-1).tolist() == [True, True, True, False, False, False]
    assert O.rownorm_global_select(np.random.default_rng(1).standard_normal((4, 3)), 1.0)[0].all()
    with pytest.raises(ValueError):
        O.rownorm_global_select(np.zeros((2, 2)), 0.0)
    with pytest.raises(ValueError):
        O.rownorm_global_select(np.zeros((2, 2)), float("nan"))


# ---------------------------------------------------------------- attention

def _sdpa(Qh, Kh, Vh, allow, scale):
    q = torch.from_numpy(Qh)[None, None]
    k = torch.from_numpy(Kh)[None, None]
    v = torch.from_numpy(Vh)[None, None]
    m = torch.from_numpy(allow)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)[0, 0]


def _case(seed, grid=(4, 4, 4), box=(2, 2, 2), n_h=2, d=8, tau=0.3):
    T, H, W = grid
    s = T * H * W
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((s, n_h, d))
    K = rng.standard_normal((s, n_h, d))
    V = rng.standard_normal((s, n_h, d))
    dO = rng.standard_normal((s, n_h, d))
    scale = 1.0 / math.sqrt(d)
    B = O.pool_blocks(K, T, H, W, box)
    S = O.block_scores(Q, B, scale)
    sel, _ = O.select_all_heads(S, tau)
    blk = O.block_of_token(T, H, W, box)
    return Q, K, V, dO, sel, blk, scale


def test_full_selection_equals_dense_sdpa():
    Q, K, V, dO, sel, blk, scale = _case(0, tau=1.0)
    assert sel.all()
    Ob, lse = O.attention_fwd(Q, K, V, sel, blk, scale)
    for h in range(Q.shape[1]):
        ref = _sdpa(Q[:, h], K[:, h], V[:, h], np.ones((Q.shape[0],) * 2, bool), scale).numpy()
        np.testing.assert_allclose(Ob[:, h], ref, rtol=1e-12, atol=1e-12)
        logits = scale * torch.from_numpy(Q[:, h]) @ torch.from_numpy(K[:, h]).T
        np.testing.assert_allclose(lse[h], torch.logsumexp(logits, 1).numpy(), rtol=1e-12)


@pytest.mark.parametrize("tau", [0.1, 0.3, 0.6])
def test_masked_attention_equals_sdpa_with_mask(tau):
    Q, K, V, dO, sel, blk, scale = _case(1, tau=tau)
    Ob, lse = O.attention_fwd(Q, K, V, sel, blk, scale, chunk=17)
    s = Q.shape[0]
    for h in range(Q.shape[1]):
        allow = sel[h][:, blk]
        has = allow.any(1)
        assert (~has).any() or tau > 0.5
        safe = allow.copy()
        safe[~has] = True                       # torch gives NaN on empty rows
        ref = _sdpa(Q[:, h], K[:, h], V[:, h], safe, scale).numpy()
        np.testing.assert_allclose(Ob[has, h], ref[has], rtol=1e-12, atol=1e-12)
        assert np.all(Ob[~has, h] == 0) and np.all(np.isneginf(lse[h][~has]))
        logits = scale * torch.from_numpy(Q[:, h]) @ torch.from_numpy(K[:, h]).T
        logits[~torch.from_numpy(allow)] = -torch.inf
        np.testing.assert_allclose(lse[h][has], torch.logsumexp(logits, 1).numpy()[has], rtol=1e-12)
    assert s == 64


@pytest.mark.parametrize("tau", [0.3, 1.0])
def test_backward_equals_torch_autograd(tau):
    Q, K, V, dO, sel, blk, scale = _case(2, tau=tau)
    dQ, dK, dV = O.attention_bwd(Q, K, V, sel, blk, scale, dO, chunk=20)
    for h in range(Q.shape[1]):
        allow = sel[h][:, blk]
        has = allow.any(1)
        safe = allow.copy()
        safe[~has] = True
        q = torch.from_numpy(Q[:, h].copy()).requires_grad_()
        k = torch.from_numpy(K[:, h].copy()).requires_grad_()
        v = torch.from_numpy(V[:, h].copy()).requires_grad_()
        out = torch.nn.functional.scaled_dot_product_attention(
            q[None, None], k[None, None], v[None, None],
            attn_mask=torch.from_numpy(safe)[None, None], scale=scale)[0, 0]
        g = torch.from_numpy(dO[:, h] * has[:, None])   # empty rows carry no gradient
        out.backward(g)
        np.testing.assert_allclose(dQ[has, h], q.grad.numpy()[has], rtol=1e-10, atol=1e-12)
        assert np.all(dQ[~has, h] == 0)
        np.testing.assert_allclose(dK[:, h], k.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dV[:, h], v.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("tau", [0.05, 0.3, 1.0])
def test_block_keys_backward_equals_full_backward(tau):
    """The per-block dK/dV evaluation (sums grouped by block, masked keys never
    formed) gives attention_bwd's rows for every block, including blocks no
    query selected (zeros), and torch autograd's key gradients."""
    Q, K, V, dO, sel, blk, scale = _case(5, tau=tau)
    dQ, dK, dV = O.attention_bwd(Q, K, V, sel, blk, scale, dO, chunk=13)
    n_b = sel.shape[2]
    seen_empty = False
    for h in range(Q.shape[1]):
        allow = sel[h][:, blk]
        safe = allow.copy()
        safe[~allow.any(1)] = True
        k = torch.from_numpy(K[:, h].copy()).requires_grad_()
        v = torch.from_numpy(V[:, h].copy()).requires_grad_()
        out = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[:, h].copy())[None, None], k[None, None], v[None, None],
            attn_mask=torch.from_numpy(safe)[None, None], scale=scale)[0, 0]
        out.backward(torch.from_numpy(dO[:, h] * allow.any(1)[:, None]))
        for j in range(n_b):
            keys, dk, dv = O.attention_bwd_block_keys(Q[:, h], K[:, h], V[:, h], sel[h], blk,
                                                      scale, dO[:, h], j)
            assert np.array_equal(keys, np.flatnonzero(blk == j))
            np.testing.assert_allclose(dk, dK[keys, h], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dv, dV[keys, h], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dk, k.grad.numpy()[keys], rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(dv, v.grad.numpy()[keys], rtol=1e-10, atol=1e-12)
            if not sel[h][:, j].any():
                seen_empty = True
                assert not dk.any() and not dv.any()
    assert seen_empty or tau > 0.1


def test_backward_central_differences():
    Q, K, V, dO, sel, blk, scale = _case(3, grid=(2, 2, 4), box=(1, 2, 2), n_h=1, d=4, tau=0.4)
    dQ, dK, dV = O.attention_bwd(Q, K, V, sel, blk, scale, dO)

    def loss(Q_, K_, V_):
        Ob, _ = O.attention_fwd(Q_, K_, V_, sel, blk, scale)
        return float(np.sum(dO * Ob))

    eps = 1e-6
    rng = np.random.default_rng(9)
    for X, G in ((Q, dQ), (K, dK), (V, dV)):
        for _ in range(6):
            idx = tuple(rng.integers(0, n) for n in X.shape)
            Xp = X.copy()
            Xm = X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p = [Xp if Y is X else Y for Y in (Q, K, V)]
            args_m = [Xm if Y is X else Y for Y in (Q, K, V)]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - G[idx]) < 1e-7 + 1e-6 * abs(fd)


def test_gradient_identities():
    # logits are bilinear in (q, k): sum_i q_i.dQ_i = sum_n k_n.dK_n, and
    # softmax rows sum to one: sum_n dK_n = 0, sum_n dV_n = sum of dO over non-empty rows
    Q, K, V, dO, sel, blk, scale = _case(4, tau=0.35)
    dQ, dK, dV = O.attention_bwd(Q, K, V, sel, blk, scale, dO)
    for h in range(Q.shape[1]):
        has = sel[h][:, blk].any(1)
        assert math.isclose(np.sum(Q[:, h] * dQ[:, h]), np.sum(K[:, h] * dK[:, h]),
                            rel_tol=1e-10, abs_tol=1e-12)
        np.testing.assert_allclose(dK[:, h].sum(0), 0.0, atol=1e-12)
        np.testing.assert_allclose(dV[:, h].sum(0), dO[has, h].sum(0), rtol=1e-12, atol=1e-12)


# -------------------------------------------------------- whole-layer cases

def test_layer_block_size_one_is_token_level_thresholding():
    T, H, W, n_h, d = 2, 3, 4, 1, 6
    s = T * H * W
    rng = np.random.default_rng(11)
    Q, K, V = (rng.standard_normal((s, n_h, d)) for _ in range(3))
    out = O.vmoba_layer(Q, K, V, T, H, W, 2, (1, 1, 1), tau=0.4)
    logits = (Q[:, 0] @ K[:, 0].T) / math.sqrt(d)
    np.testing.assert_allclose(out["S"][0], logits, rtol=1e-12, atol=1e-13)
    # token-level: each selected (query, key) pair is one of the top logits
    sel = out["sel"][0]
    assert logits[sel].min() >= logits[~sel].max()


def test_layer_single_block_is_all_or_nothing_per_row():
    T, H, W, n_h, d = 2, 2, 4, 1, 4
    s = T * H * W
    rng = np.random.default_rng(12)
    Q, K, V = (rng.standard_normal((s, n_h, d)) for _ in range(3))
    out = O.vmoba_layer(Q, K, V, T, H, W, 0, (2, 2, 4), tau=0.5)
    assert out["sel"].shape == (1, s, 1)
    has = out["sel"][0, :, 0]
    dense = _sdpa(Q[:, 0], K[:, 0], V[:, 0], np.ones((s, s), bool), 1 / math.sqrt(d)).numpy()
    np.testing.assert_allclose(out["O"][has, 0], dense[has], rtol=1e-12, atol=1e-12)
    assert np.all(out["O"][~has, 0] == 0)
    # the selected rows are those with the largest q . mean(K)
    qb = Q[:, 0] @ K[:, 0].mean(0)
    assert qb[has].min() >= qb[~has].max()


def test_layer_full_threshold_is_dense_attention_on_workload_inputs():
    w = synth.WORKLOADS[1]
    q, k, v = synth.make_qkv(w.wid, 0, w.T, w.H, w.W, w.n_heads, w.head_dim, kind=w.kind)
    for mode in range(3):
        out = O.vmoba_layer(q, k, v, w.T, w.H, w.W, mode, w.boxes[mode], tau=1.0)
        assert out["sel"].all()
        for h in range(w.n_heads):
            ref = _sdpa(q[:, h], k[:, h], v[:, h], np.ones((w.s, w.s), bool),
                        1 / math.sqrt(w.head_dim)).numpy()
            np.testing.assert_allclose(out["O"][:, h], ref, rtol=1e-11, atol=1e-12)


def test_round_io_matches_torch_casts():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.standard_normal(4096) * 10.0 ** rng.integers(-6, 6, 4096),
                        [0.0, -0.0, 1.0, 2.0 ** -130, 3.0e38, -np.inf, np.inf]])
    for dt, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        ref = torch.from_numpy(x).to(torch.float32).to(tdt).to(torch.float64).numpy()
        got = O.round_io(x, dt)
        np.testing.assert_array_equal(got, ref)


def test_half_ulp_bounds_the_rounding_of_torch_casts():
    rng = np.random.default_rng(22)
    x = rng.standard_normal(20000) * 10.0 ** rng.integers(-5, 5, 20000)
    for dt, tdt in (("bf16", torch.bfloat16), ("f32", torch.float32)):
        stored = torch.from_numpy(x).to(torch.float32).to(tdt).to(torch.float64).numpy()
        assert O.io_excess_error(stored, x, dt) == 0.0
        # one ulp off is detected
        bumped = stored + 4.0 * O.io_half_ulp(x, dt)
        assert O.io_excess_error(bumped, x, dt) > 0.0
