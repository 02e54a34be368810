"""The bench's FLOP convention against the FLOP columns the pages print.

tests/golden/flops_tables.json holds the VMoBA notes' Table 2 / Table 1
numbers.  With 4*d FLOPs per attended token pair per head (so 4*s^2*D per
dense layer forward) and the printed "sparsity" read as the fraction of
token pairs attended, the sparse rows follow from the full-attention rows to
within half a percent.  A different per-pair count (e.g. 2*d) or reading
sparsity as the fraction dropped fails this test.
"""
import json
import os

import pytest

from block_sparse_attention_layer_b200 import metrics

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "flops_tables.json")
DATA = json.load(open(GOLDEN))


@pytest.mark.parametrize("row", DATA["rows"], ids=lambda r: f"{r['table']}-{r['video']}-{r['method']}")
def test_sparse_flops_follow_from_density(row):
    layers = DATA["model"]["layers"]
    D = DATA["model"]["model_dim"]
    T, H, W = row["latent"]
    s = T * H * W
    # dense attention of one model forward: every (query, key) pair, all heads
    head_dim = 128
    n_heads = D // head_dim
    attn_dense = layers * n_heads * metrics.attention_flops(s * s, head_dim) / 1e12
    linear = row["full_tflops"] - attn_dense
    assert 0.15 < linear / row["full_tflops"] < 0.25        # the non-attention part of the model
    pairs = row["sparsity"] * s * s
    predicted = linear + layers * n_heads * metrics.attention_flops(pairs, head_dim) / 1e12
    assert abs(predicted - row["sparse_tflops"]) / row["sparse_tflops"] < DATA["tolerance_rel"]


def test_backward_convention():
    assert metrics.attention_flops(1, 128, forward=True, backward=True) == 14 * 128
    assert metrics.token_pairs_from_stats([3, 4], 192) == 7 * 192
