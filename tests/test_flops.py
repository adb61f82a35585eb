"""Analytic counters: exact kept-FLOP count on a brute-force mask, and the pages' FLOP claims."""
import numpy as np

from sparse_rank_hybrid_b200 import flops as F
from sparse_rank_hybrid_b200 import workloads as W


def test_sparse_flops_brute_force():
    rng = np.random.default_rng(0)
    L, b, D = 300, 64, 16
    nb = 5
    idx = np.stack([rng.choice(nb, 2, replace=False) for _ in range(nb)])[None]
    # brute force over (query, key) pairs allowed by the mask
    allowed = 0
    for i in range(L):
        for j in range(L):
            allowed += (j // b) in idx[0, i // b]
    assert F.sparse_flops(idx, L, b, D) == 4 * D * allowed


def test_up_to_10x_fewer_flops_at_90_percent_sparsity():
    """RoPeSLR abstract: up to 10x fewer FLOPs on Wan2.1-1.3B at 90% sparsity.  With the kept
    sparse work plus the low-rank branch at r = 32 the ratio to dense attention is just under 10."""
    w = W.WAN_1_3B
    BH = w.heads
    kept = F.sparse_flops_nominal(w.L, w.block, w.head_dim, BH, 26)
    hybrid = kept + F.lowrank_flops(w.L, w.rank, w.head_dim, BH)
    ratio = F.dense_flops(w.L, w.head_dim, BH) / hybrid
    assert 9.0 < ratio < 10.0


def test_lowrank_matches_full_width_linear_at_half_rank():
    """RoLA App. F: at r = d_h / 2 the low-rank branch's leading matmul FLOPs equal a full-width
    linear-attention branch's (4 L d_h^2 per head, RoPeSLR appendix FLOP analysis)."""
    L, D = 32760, 128
    assert F.lowrank_flops(L, D // 2, D, 1) == 4 * L * D * D
