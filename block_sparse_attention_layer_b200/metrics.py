"""FLOP and byte accounting for the throughput numbers.

FLOP convention (pinned against the FLOP columns of the VMoBA notes'
Table 1 and Table 2, which it reproduces to a fraction of a percent from the
full-attention row and the printed sparsity): one attended (query, key)
token pair of one head costs 4*d FLOPs in the forward pass (q.k and p*v,
a multiply and an add each) and 10*d in the backward pass (S recompute,
dP = dO V^T, dV += P^T dO, dK += dS^T Q, dQ += dS K).  Only selected pairs
count; work a kernel spends on masked-out positions does not.
"""
from __future__ import annotations

FWD_FLOPS_PER_PAIR_PER_DIM = 4
BWD_FLOPS_PER_PAIR_PER_DIM = 10


def attention_flops(token_pairs: float, head_dim: int, forward: bool = True,
                    backward: bool = False) -> float:
    """FLOPs of sparse attention over ``token_pairs`` attended (query, key) pairs."""
    per = 0
    if forward:
        per += FWD_FLOPS_PER_PAIR_PER_DIM
    if backward:
        per += BWD_FLOPS_PER_PAIR_PER_DIM
    return float(token_pairs) * per * head_dim


def token_pairs_from_stats(n_selected_per_head, block_len: int) -> int:
    """Attended token pairs: each selected (query, block) pair covers block_len keys."""
    return int(sum(int(n) for n in n_selected_per_head)) * int(block_len)


def partition_bytes(s: int, n_heads: int, head_dim: int, elem: int, n_blocks: int) -> int:
    """Declared traffic of the partition kernel: read K, V; write K', V'; write B (fp32)."""
    return 4 * s * n_heads * head_dim * elem + n_heads * n_blocks * head_dim * 4


def select_bytes(s: int, n_heads: int, n_blocks: int) -> int:
    """Algorithmic traffic of selection: one read of the fp32 pool + the bitmap write."""
    words = (n_blocks + 31) // 32
    return s * n_heads * n_blocks * 4 + s * n_heads * words * 4
