"""Plain fp64 CPU oracle of VMoBA per-layer sparse attention.

TEST INFRASTRUCTURE ONLY.  This module defines what the CUDA library must
compute, step by step and in float64, so that the kernels can be checked
against it.  Only the test suite, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the library itself never does
and shares no code with it.

Sources (VMoBA: Mixture-of-Block Attention for Video Diffusion Models):

* [notes] papernotes.org ICLR 2026 notes, section "Method / overall
  framework" and "Key designs" 1-3 (the only page with the formulas);
* [digest] paperlayer.ai section digest of arXiv 2506.23858, sections
  3.1-3.4.

Every function below names the passage it follows.  Where the pages leave a
step open, the reading taken is stated in the function's docstring:

1. "Normalised similarity" (notes, key design 3; digest 3.4) is read as a
   softmax over the head's whole s x N_b pool of scores S = scale * q . b,
   scale = 1/sqrt(head_dim).  Every term is >= 0, the total is 1 so tau is
   the fraction of similarity mass kept, and the order equals the order of S.
2. The stopping rule uses ">=" (the printed formula), not "exceeds".
3. Ties in the ranking are broken by (query index asc, block index asc).
4. tau at or above the pool's total mass selects every pair.
5. A query row with no selected block gets O = 0, LSE = -inf, dQ = 0.
6. K and V are permuted together; Q and the output keep the original order.
7. Blocks are numbered row-major over the (T/bt, H/bh, W/bw) grid and
   tokens inside a block are in (t, y, x) order.
8. The selection mask is a constant for the backward pass (no gradient
   flows through the pooled blocks or the threshold).
9. O, dQ, dK, dV are returned in the I/O dtype, rounded to nearest from the
   exact values; LSE stays fp32.  The storage rounding (up to half an ulp of
   the result: 0.03 at |x| = 9 in bf16) is not an error of the computation,
   so tolerances apply to |stored - exact| - half_ulp(exact) (io_excess_error);
   round_io gives the rounded exact value itself.
10. The ablation's selection variants (notes, ablation table rows "topk +
    global", "threshold + local", "topk + local (about MoBA's selection)";
    digest App. A, training-free runs: 3D blocks with MoBA's local top-k):
    "local" normalises each query row's own N_b scores with a softmax at the
    same temperature and selects per row; "top-k" keeps a fixed count -- k
    pairs of the head's pool (global) or k blocks per query row (local) --
    ranked like the method, ties by index.  The pages give no k; it is a
    parameter here.
11. The other reading of "normalised similarity", rejected for the method
    and kept as a variant: each query's scores are normalised by a softmax
    over that query's own N_b blocks and divided by s, so every query row
    carries mass 1/s of the head's total 1; the head's whole pool is ranked
    by that value (ties by query, then block) and key design 3's cumulative
    rule is applied to it.

Pins (what ties each function to something other than itself) are in
``tests/test_oracle_pins.py``; each function's docstring lists them.

Array conventions: Q, K, V, O, dO, dQ, dK, dV are ``[s][n_heads][d]``
float64 in original token order ``t*H*W + y*W + x``.
"""
from __future__ import annotations

import math

import numpy as np

MODES = {0: "1D", 1: "2D", 2: "3D"}


# --------------------------------------------------------------------------
# Partition (notes, key design 1: layer-wise recurrent 1D-2D-3D partition)
# --------------------------------------------------------------------------

def mode_for_layer(layer: int) -> int:
    """Partition mode of layer l: l mod 3 = 0 -> 1D, 1 -> 2D, 2 -> 3D.

    [notes] key design 1; [digest] 3.2.  Pinned: tests check the cycle.
    """
    if layer < 0:
        raise ValueError("layer index must be >= 0")
    return layer % 3


def mode_box(mode: int, T: int, H: int, W: int, bt: int, bh: int, bw: int) -> tuple:
    """Block box of a mode.

    [notes] key design 1: 1D groups tokens of adjacent frames (box bt x H x W);
    2D groups tokens of one spatial region across all frames (T x bh x bw);
    3D cuts local spatio-temporal patches (bt x bh x bw).
    """
    if mode == 0:
        return (bt, H, W)
    if mode == 1:
        return (T, bh, bw)
    if mode == 2:
        return (bt, bh, bw)
    raise ValueError(f"mode must be 0, 1 or 2, got {mode}")


def check_box(T: int, H: int, W: int, box: tuple) -> None:
    bt, bh, bw = box
    if min(bt, bh, bw) < 1 or T % bt or H % bh or W % bw:
        raise ValueError(f"box {box} does not divide the latent {(T, H, W)}")


def partition_order(T: int, H: int, W: int, box: tuple) -> np.ndarray:
    """Key permutation of the partition: K'[p] = K[perm[p]].

    [notes] key design 1 writes the partition as a rearrange of K in (T H W)
    order; read here as (pt bt)(ph bh)(pw bw) -> (pt ph pw)(bt bh bw), i.e.
    blocks row-major over the box grid, (t, y, x) order inside a block.
    Pinned: brute-force coordinate enumeration; 3D boxes that equal a 1D or
    2D box give the same partition; every block holds one box of tokens.
    """
    check_box(T, H, W, box)
    bt, bh, bw = box
    idx = np.arange(T * H * W).reshape(T // bt, bt, H // bh, bh, W // bw, bw)
    return idx.transpose(0, 2, 4, 1, 3, 5).reshape(-1).copy()


def block_of_token(T: int, H: int, W: int, box: tuple) -> np.ndarray:
    """Block index of every original token (inverse view of partition_order)."""
    perm = partition_order(T, H, W, box)
    L = box[0] * box[1] * box[2]
    blk = np.empty(T * H * W, dtype=np.int64)
    blk[perm] = np.arange(perm.size) // L
    return blk


def permute_keys(K: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """K' = rearranged K, returned as [n_heads][s][d] (block-contiguous)."""
    return np.ascontiguousarray(K[perm].transpose(1, 0, 2))


def pool_blocks(K: np.ndarray, T: int, H: int, W: int, box: tuple) -> np.ndarray:
    """Block tensor B = mean(K') per block, [n_heads][N_b][d].

    [notes] key design 1: B = mean(K') over each block of the rearranged keys.
    Pinned: brute-force coordinate sums; constant keys give B = K; the mean
    of the block means equals the mean of all keys.
    """
    perm = partition_order(T, H, W, box)
    L = box[0] * box[1] * box[2]
    Kp = permute_keys(K, perm)
    n_h, s, d = Kp.shape
    return Kp.reshape(n_h, s // L, L, d).mean(axis=2)


# --------------------------------------------------------------------------
# Scores (notes, key design 2: global block selection, S = q_i b_i^T)
# --------------------------------------------------------------------------

def block_scores(Q: np.ndarray, B: np.ndarray, scale: float) -> np.ndarray:
    """Pool of head i: S_i = scale * q_i b_i^T, returned as [n_heads][s][N_b].

    [notes] key design 2 (M_i = TopkMask(q_i b_i^T, k)) and key design 3
    (S^ = q_i b_i^T); the 1/sqrt(d) temperature is reading 1.
    Pinned: equals the block-average of the token-level logits (linearity of
    the mean), computed from the full logit matrix.
    """
    Qh = Q.transpose(1, 0, 2)                      # [n_h][s][d]
    return scale * np.matmul(Qh, B.transpose(0, 2, 1))


# --------------------------------------------------------------------------
# Threshold selection (notes, key design 3; digest 3.3 and 3.4)
# --------------------------------------------------------------------------

def normalised_pool(S_h: np.ndarray) -> np.ndarray:
    """p = exp(S - max S) / sum exp(S - max S) over the head's whole pool (reading 1)."""
    e = np.exp(S_h - S_h.max())
    return e / e.sum()


def threshold_select(S_h: np.ndarray, tau: float):
    """Global threshold selection for one head.

    [notes] key design 3: sort the global pool descending and take
    k = min{k' : sum_{j<=k'} Sorted(S^)_j >= tau} over normalised similarity;
    [digest] 3.4 says the same in words.  Ties: (query asc, block asc).

    Returns (mask [s][N_b] bool, stats) with stats = dict(k, cut_score, mass)
    where mass is the cumulative normalised mass of the k selected pairs.
    Pinned: minimality (c_k >= tau > c_{k-1}), density bound
    k/(s N_b) < tau + 1/(s N_b), monotonicity in tau, brute-force subset
    enumeration on tiny pools, and the selected set scoring at least as high
    as every unselected pair.
    """
    if not (tau > 0.0) or math.isnan(tau):
        raise ValueError("tau must be > 0")
    flat = S_h.reshape(-1)
    p = normalised_pool(S_h).reshape(-1)
    order = np.argsort(-flat, kind="stable")       # descending, ties by flat index
    c = np.cumsum(p[order])
    reached = np.flatnonzero(c >= tau)
    k = int(reached[0]) + 1 if reached.size else flat.size
    mask = np.zeros(flat.size, dtype=bool)
    mask[order[:k]] = True
    stats = dict(k=k, cut_score=float(flat[order[k - 1]]), mass=float(c[k - 1]))
    return mask.reshape(S_h.shape), stats


def select_all_heads(S: np.ndarray, tau: float):
    """threshold_select for every head: mask [n_heads][s][N_b], list of stats."""
    masks, stats = [], []
    for h in range(S.shape[0]):
        m, st = threshold_select(S[h], tau)
        masks.append(m)
        stats.append(st)
    return np.stack(masks), stats


# --------------------------------------------------------------------------
# Selection variants of the ablation (notes, ablation table: the method is
# "threshold + global"; the other rows replace the threshold by a fixed
# count, the global pool by per-query selection, or both; digest App. A)
# --------------------------------------------------------------------------

def topk_global_select(S_h: np.ndarray, k: int):
    """"topk + global": the k pairs of the head's whole pool ranked first by
    (S desc, query asc, block asc) -- the method's ranking with a fixed count
    in place of the mass threshold (reading 10).

    Returns (mask [s][N_b] bool, stats) with stats = dict(k, cut_score, mass),
    mass under the head's pool normalisation (reading 1).
    Pinned: equals threshold_select when k is that selection's k*; the kept
    set has the largest score sum of all k-subsets (brute force on tiny
    pools); nested in k; a constant pool keeps the first k flat indices.
    """
    if not (k >= 1) or int(k) != k:
        raise ValueError("k must be a positive integer")
    flat = S_h.reshape(-1)
    k = min(int(k), flat.size)
    order = np.argsort(-flat, kind="stable")
    mask = np.zeros(flat.size, dtype=bool)
    mask[order[:k]] = True
    p = normalised_pool(S_h).reshape(-1)
    stats = dict(k=k, cut_score=float(flat[order[k - 1]]), mass=float(p[order[:k]].sum()))
    return mask.reshape(S_h.shape), stats


def _row_softmax(row: np.ndarray) -> np.ndarray:
    e = np.exp(row - row.max())
    return e / e.sum()


def rownorm_global_select(S_h: np.ndarray, tau: float):
    """"threshold + global" under the per-query reading of the normalised
    similarity (reading 11): p_ij = softmax_j(S_i.) / s over the head's whole
    pool, ranked by p descending (ties: query asc, block asc); keep the
    shortest prefix whose mass reaches tau (every pair if rounding leaves the
    total short) -- key design 3's rule on this normalisation.

    Returns (mask [s][N_b] bool, stats) with stats = dict(k, cut_logp, mass):
    cut_logp = S_ij - logsumexp_j' S_ij' of the last kept pair (its log row
    softmax), mass = the kept p.
    Pinned: one query row, and a pool whose rows are all equal, give
    threshold_select's set; invariant under adding a constant to a row
    (threshold_select is not); brute-force subset enumeration on tiny pools;
    minimality.
    """
    if not (tau > 0.0) or math.isnan(tau):
        raise ValueError("tau must be > 0")
    s, nb = S_h.shape
    logp = np.empty((s, nb))
    for i in range(s):
        m = S_h[i].max()
        logp[i] = S_h[i] - (m + math.log(np.exp(S_h[i] - m).sum()))
    flat = logp.reshape(-1)
    p = np.exp(flat) / s
    order = np.argsort(-flat, kind="stable")       # descending, ties by flat index
    c = np.cumsum(p[order])
    reached = np.flatnonzero(c >= tau)
    k = int(reached[0]) + 1 if reached.size else flat.size
    mask = np.zeros(flat.size, dtype=bool)
    mask[order[:k]] = True
    stats = dict(k=k, cut_logp=float(flat[order[k - 1]]), mass=float(c[k - 1]))
    return mask.reshape(S_h.shape), stats


def threshold_local_select(S_h: np.ndarray, tau: float):
    """"threshold + local": per query row, p = softmax of the row's own N_b
    scores; rank the row's blocks (S desc, block asc) and keep the shortest
    prefix whose mass reaches tau (every block if rounding leaves the total
    short) -- key design 3's rule applied to one row (reading 10).

    Returns (mask, stats) with stats = dict(k (pairs), cut_scores [s] (score
    of each row's last kept block), mass (mean kept mass per row)).
    Pinned: one query row equals threshold_select; per-row minimality
    (kept mass >= tau > mass without the last block); the kept set has the
    fewest blocks reaching tau and the largest mass among such sets (brute
    force on tiny rows); every row keeps >= 1 block.
    """
    if not (tau > 0.0) or math.isnan(tau):
        raise ValueError("tau must be > 0")
    s, nb = S_h.shape
    mask = np.zeros((s, nb), dtype=bool)
    cuts = np.empty(s)
    kept = np.empty(s)
    for i in range(s):
        p = _row_softmax(S_h[i])
        order = np.argsort(-S_h[i], kind="stable")
        c = np.cumsum(p[order])
        reached = np.flatnonzero(c >= tau)
        k = int(reached[0]) + 1 if reached.size else nb
        mask[i, order[:k]] = True
        cuts[i] = S_h[i, order[k - 1]]
        kept[i] = c[k - 1]
    return mask, dict(k=int(mask.sum()), cut_scores=cuts, mass=float(kept.mean()))


def topk_local_select(S_h: np.ndarray, k: int):
    """"topk + local" (about MoBA's selection): each query row keeps its
    min(k, N_b) blocks ranked first by (S desc, block asc) (reading 10).

    Returns (mask, stats) as threshold_local_select, mass under the row
    softmax.  Pinned: every row keeps exactly min(k, N_b); one query row
    equals topk_global_select; the kept blocks have the largest score sum of
    all k-subsets of the row (brute force on tiny rows).
    """
    if not (k >= 1) or int(k) != k:
        raise ValueError("k must be a positive integer")
    s, nb = S_h.shape
    k = min(int(k), nb)
    mask = np.zeros((s, nb), dtype=bool)
    cuts = np.empty(s)
    kept = np.empty(s)
    for i in range(s):
        order = np.argsort(-S_h[i], kind="stable")
        mask[i, order[:k]] = True
        cuts[i] = S_h[i, order[k - 1]]
        kept[i] = _row_softmax(S_h[i])[order[:k]].sum()
    return mask, dict(k=int(mask.sum()), cut_scores=cuts, mass=float(kept.mean()))


# --------------------------------------------------------------------------
# Sparse attention over the selected pairs (notes, overall framework:
# "attention only on the selected blocks, same shape as full attention")
# --------------------------------------------------------------------------

def allowed_keys(sel_h: np.ndarray, blk: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Token-level mask [len(rows)][s]: key n allowed for row i iff block(n) is selected."""
    return sel_h[rows][:, blk]


def attention_fwd_rows(Qh, Kh, Vh, sel_h, blk, scale, rows):
    """Forward of the masked softmax attention for the given query rows of one head.

    Definition (reading 5 for empty rows): a_in = scale q_i.k_n over keys whose
    block is selected for row i; LSE_i = log sum exp a_in; O_i = softmax(a_i) V.
    Pinned: tau = 1 equals torch's scaled_dot_product_attention in fp64; any
    mask equals SDPA with the same boolean mask on non-empty rows.
    Returns O [len(rows)][d], LSE [len(rows)].
    """
    A = scale * (Qh[rows] @ Kh.T)
    allow = allowed_keys(sel_h, blk, rows)
    A = np.where(allow, A, -np.inf)
    has = allow.any(axis=1)
    m = np.where(has, A.max(axis=1), 0.0)
    P = np.exp(A - m[:, None])                      # exp(-inf) = 0 on masked keys
    l = P.sum(axis=1)
    O = np.zeros((len(rows), Vh.shape[1]))
    O[has] = (P[has] @ Vh) / l[has, None]
    lse = np.full(len(rows), -np.inf)
    lse[has] = m[has] + np.log(l[has])
    return O, lse


def attention_bwd_rows(Qh, Kh, Vh, sel_h, blk, scale, rows, dOh_rows):
    """Backward for a chunk of query rows of one head, mask held constant (reading 8).

    With P the masked softmax, D_i = dO_i . O_i, dP = dO V^T,
    dS = P * (dP - D), the chunk contributes dQ_rows = scale dS K,
    dK += scale dS^T Q_rows, dV += P^T dO_rows.
    Pinned: central finite differences of sum(dO * O) in fp64 and torch
    autograd through SDPA with the same boolean mask.
    Returns (dQ_rows, dK_part, dV_part).
    """
    A = scale * (Qh[rows] @ Kh.T)
    allow = allowed_keys(sel_h, blk, rows)
    A = np.where(allow, A, -np.inf)
    has = allow.any(axis=1)
    m = np.where(has, A.max(axis=1), 0.0)
    P = np.exp(A - m[:, None])
    l = P.sum(axis=1)
    P[has] /= l[has, None]
    P[~has] = 0.0
    O = P @ Vh
    D = np.sum(dOh_rows * O, axis=1)
    dP = dOh_rows @ Vh.T
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ Kh)
    dK = scale * (dS.T @ Qh[rows])
    dV = P.T @ dOh_rows
    return dQ, dK, dV


def attention_bwd_block_keys(Qh, Kh, Vh, sel_h, blk, scale, dOh, j):
    """dK and dV of block j's keys in one head (mask held constant, reading 8).

    Only the queries that selected block j reach its keys.  Each of them
    needs its LSE_i and O_i over all of its own selected keys; those sums are
    taken block by block over the blocks the query selected -- the same
    terms as attention_fwd_rows, grouped by block, with masked keys (whose
    terms are exactly 0) never formed, so the cost follows the selected pairs
    instead of s x s.  Two passes: the row maxima, then the sums.  Then for
    the keys n of block j: P_in = exp(scale q_i.k_n - LSE_i),
    D_i = dO_i . O_i, dS = P (dO_i.v_n - D_i), dK_n = scale sum_i dS_in q_i,
    dV_n = sum_i P_in dO_i.
    Pinned: equals the rows of attention_bwd's dK, dV for every block, and
    torch autograd through masked SDPA.
    Returns (keys of block j in original order, dK [len][d], dV [len][d]).
    """
    keys_j = np.flatnonzero(blk == j)
    d = Qh.shape[1]
    rows = np.flatnonzero(sel_h[:, j])
    if rows.size == 0:
        return keys_j, np.zeros((keys_j.size, d)), np.zeros((keys_j.size, d))
    n_blocks = sel_h.shape[1]
    members = [np.flatnonzero(blk == b) for b in range(n_blocks)]
    sub = sel_h[rows]
    m = np.full(rows.size, -np.inf)
    for b in range(n_blocks):
        r = np.flatnonzero(sub[:, b])
        if r.size:
            m[r] = np.maximum(m[r], (scale * (Qh[rows[r]] @ Kh[members[b]].T)).max(axis=1))
    l = np.zeros(rows.size)
    O = np.zeros((rows.size, d))
    for b in range(n_blocks):
        r = np.flatnonzero(sub[:, b])
        if r.size:
            P = np.exp(scale * (Qh[rows[r]] @ Kh[members[b]].T) - m[r, None])
            l[r] += P.sum(axis=1)
            O[r] += P @ Vh[members[b]]
    O /= l[:, None]
    lse = m + np.log(l)
    P = np.exp(scale * (Qh[rows] @ Kh[keys_j].T) - lse[:, None])
    dO = dOh[rows]
    D = np.sum(dO * O, axis=1)
    dS = P * (dO @ Vh[keys_j].T - D[:, None])
    return keys_j, scale * (dS.T @ Qh[rows]), P.T @ dO


def _row_chunks(s: int, chunk: int):
    for r0 in range(0, s, chunk):
        yield np.arange(r0, min(s, r0 + chunk))


def attention_fwd(Q, K, V, sel, blk, scale, chunk: int = 1024):
    """Masked attention forward for all heads: O [s][n_h][d], LSE [n_h][s]."""
    s, n_h, d = Q.shape
    O = np.zeros_like(Q)
    lse = np.zeros((n_h, s))
    for h in range(n_h):
        for rows in _row_chunks(s, chunk):
            o, l_ = attention_fwd_rows(Q[:, h], K[:, h], V[:, h], sel[h], blk, scale, rows)
            O[rows, h] = o
            lse[h, rows] = l_
    return O, lse


def attention_bwd(Q, K, V, sel, blk, scale, dO, chunk: int = 1024):
    """Masked attention backward for all heads: dQ, dK, dV in [s][n_h][d]."""
    s, n_h, d = Q.shape
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for h in range(n_h):
        for rows in _row_chunks(s, chunk):
            dq, dk, dv = attention_bwd_rows(Q[:, h], K[:, h], V[:, h], sel[h], blk,
                                            scale, rows, dO[rows, h])
            dQ[rows, h] = dq
            dK[:, h] += dk
            dV[:, h] += dv
    return dQ, dK, dV


# --------------------------------------------------------------------------
# The whole layer (notes, overall framework flowchart; digest 3.1)
# --------------------------------------------------------------------------

def vmoba_layer(Q, K, V, T, H, W, mode, box_cfg, tau, scale=None, dO=None,
                chunk: int = 1024):
    """Partition -> pool -> scores -> global threshold selection -> attention.

    ``box_cfg`` is (bt, bh, bw); ``mode`` picks which of its axes apply
    (mode_box).  Returns a dict with perm, blk, B, S, sel, stats, O, LSE and,
    when dO is given, dQ, dK, dV.
    """
    s, n_h, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    box = mode_box(mode, T, H, W, *box_cfg)
    perm = partition_order(T, H, W, box)
    blk = block_of_token(T, H, W, box)
    B = pool_blocks(K, T, H, W, box)
    S = block_scores(Q, B, scale)
    sel, stats = select_all_heads(S, tau)
    O, lse = attention_fwd(Q, K, V, sel, blk, scale, chunk)
    out = dict(box=box, perm=perm, blk=blk, B=B, S=S, sel=sel, stats=stats,
               O=O, LSE=lse, scale=scale)
    if dO is not None:
        dQ, dK, dV = attention_bwd(Q, K, V, sel, blk, scale, dO, chunk)
        out.update(dQ=dQ, dK=dK, dV=dV)
    return out


def round_io(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round exact results to the layer's I/O dtype (reading 9), back as float64.

    fp32: IEEE round-to-nearest-even.  bf16: the fp32 value's upper 16 bits
    rounded to nearest-even.  Pinned against torch's float -> bfloat16 cast.
    """
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x32.astype(np.float64)
    bits = np.ascontiguousarray(x32).view(np.uint32).astype(np.uint64)
    keep = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    finite = np.isfinite(x32)
    out = np.where(finite, keep, bits >> 16).astype(np.uint32) << 16
    return out.view(np.float32).astype(np.float64)


def io_half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half an ulp of the I/O dtype at each exact value (bf16: 8, fp32: 24 significant bits)."""
    bits = 8 if dtype == "bf16" else 24
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)                       # subnormal range of both formats
    return np.where(a > 0, 2.0 ** (e - bits), 2.0 ** (-126 - bits))


def io_excess_error(stored: np.ndarray, exact: np.ndarray, dtype: str) -> float:
    """max |stored - exact| beyond the half-ulp rounding of storing ``exact`` (reading 9)."""
    err = np.abs(np.asarray(stored, np.float64) - exact) - io_half_ulp(exact, dtype)
    return float(max(err.max(), 0.0)) if err.size else 0.0

