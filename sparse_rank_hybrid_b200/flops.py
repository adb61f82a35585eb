"""Analytic work counters of the hybrid attention forward (host logic, used by the benchmark).

FLOPs (multiply-add = 2):
  sparse branch  4 * D * sum_alpha |alpha| * sum_{beta in K(alpha)} |beta|   (q k^T and p v, exactly
                 over the kept blocks, with the partial last block counted at its real size)
  low-rank       8 * L * r * D per head: the two feature products (q A, k A), the summary
                 sum_j psi_k v^T and the readout psi_q^T S (RoLA, "F Computational Complexity
                 Analysis": the branch is O(L r d_h); at r = d_h/2 it matches a full-width linear
                 branch's leading cost)
  scores         2 * nb^2 * D per head
Bytes (algorithmic minimum): q, k, v read once (bf16) + out written once.
"""
from __future__ import annotations

import numpy as np


def block_sizes(L: int, block: int) -> np.ndarray:
    nb = -(-L // block)
    s = np.full(nb, block, dtype=np.int64)
    s[-1] = L - (nb - 1) * block
    return s


def sparse_flops(idx: np.ndarray, L: int, block: int, D: int) -> float:
    """idx: [BH, nb, k] kept key blocks per query block (any order)."""
    sz = block_sizes(L, block)
    kept = sz[idx].sum(axis=-1)             # [BH, nb] keys seen by each query block
    return float(4.0 * D * (kept * sz[None, :]).sum())


def sparse_flops_nominal(L: int, block: int, D: int, BH: int, keep: int) -> float:
    """Kept FLOPs assuming full kept key blocks (upper estimate when the last block is kept)."""
    sz = block_sizes(L, block)
    return float(4.0 * D * BH * keep * block * sz.sum())


def lowrank_flops(L: int, r: int, D: int, BH: int) -> float:
    return float(8.0 * L * r * D * BH)


def score_flops(nb: int, D: int, BH: int) -> float:
    return float(2.0 * nb * nb * D * BH)


def dense_flops(L: int, D: int, BH: int) -> float:
    return float(4.0 * L * L * D * BH)


def io_bytes(B: int, L: int, Hh: int, D: int, r: int, out_bytes: int = 4) -> float:
    n = B * L * Hh * D
    return float(3 * n * 2 + n * out_bytes + D * r * 2)
