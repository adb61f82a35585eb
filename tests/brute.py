"""Independent brute-force formulations used to pin the fp64 oracle.

None of this shares code with the oracle: each function computes the same quantity another way
(complex arithmetic instead of 2x2 rotations, a dense masked attention from torch instead of the
gathered-key loop, a full lexicographic sort instead of the comparator sort, the explicit L x L
quadratic form instead of the query-independent summary).  Test-only.
"""
from __future__ import annotations

import numpy as np
import torch


def grid_positions(grid, offset=(0, 0, 0)):
    """[L, 3] integer (t, h, w) of each flattened token, via numpy's own unravel (row-major)."""
    T, H, W = grid
    t, h, w = np.unravel_index(np.arange(T * H * W), (T, H, W))
    return np.stack([t + offset[0], h + offset[1], w + offset[2]], axis=1).astype(np.float64)


def rope_complex(x, pos, axis, omega, npairs):
    """Rotate pair j of each row as the complex number x_2j + i x_2j+1 times exp(i pos_axis(j) omega_j)."""
    x = np.asarray(x, dtype=np.float64)
    z = x[:, 0:2 * npairs:2] + 1j * x[:, 1:2 * npairs:2]
    ang = pos[:, axis[:npairs]] * omega[None, :npairs]
    zr = z * np.exp(1j * ang)
    y = x.copy()
    y[:, 0:2 * npairs:2] = zr.real
    y[:, 1:2 * npairs:2] = zr.imag
    return y


def masked_dense_attention(qh, kh, v, allowed):
    """softmax(qh kh^T / sqrt(D) + mask) v with torch's fp64 SDPA; allowed [Lq, Lk] bool."""
    q = torch.from_numpy(np.ascontiguousarray(qh))[None, None]
    k = torch.from_numpy(np.ascontiguousarray(kh))[None, None]
    vv = torch.from_numpy(np.ascontiguousarray(v))[None, None]
    m = torch.from_numpy(np.ascontiguousarray(allowed))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, vv, attn_mask=m)
    return o[0, 0].numpy()


def block_mask(idx, L, block):
    """[L, L] bool: query i may see key j iff j's block is in i's block's kept list."""
    nb = idx.shape[0]
    kept = np.zeros((nb, nb), dtype=bool)
    for a in range(nb):
        kept[a, idx[a]] = True
    bl = np.arange(L) // block
    return kept[bl][:, bl]


def topk_lexsort(s, k):
    """First k of each row under (score desc, index asc) by a full lexicographic sort, ascending."""
    nb = s.shape[0]
    out = np.empty((nb, k), dtype=np.int64)
    for a in range(nb):
        order = np.lexsort((np.arange(nb), -s[a]))
        out[a] = np.sort(order[:k])
    return out


def lowrank_quadratic(psiq, phiq, psik, phik, v, eps=1e-6):
    """O_i = sum_j (psiq_i . psik_j) v_j / (sum_j phiq_i . phik_j + eps), the explicit L x L form."""
    num_w = psiq @ psik.T
    den = (phiq @ phik.T).sum(axis=1, keepdims=True) + eps
    return (num_w @ v) / den


def relative_kernel(fq, fk, pos_q, pos_k, axis, omega, npairs):
    """sum over rotated pairs of Re[(fq_j)(conj fk_j) exp(i (p_q - p_k) omega_j)] + plain dot of the rest.

    This is the value of psi(q) . psi(k) written through the position DIFFERENCE only (the relative
    property of RoPE applied outside the activation)."""
    zq = fq[..., 0:2 * npairs:2] + 1j * fq[..., 1:2 * npairs:2]
    zk = fk[..., 0:2 * npairs:2] + 1j * fk[..., 1:2 * npairs:2]
    dang = (pos_q[:, None, :][..., axis[:npairs]] - pos_k[None, :, :][..., axis[:npairs]]) * omega[:npairs]
    rot = (zq[:, None, :] * np.conj(zk[None, :, :]) * np.exp(1j * dang)).real.sum(-1)
    rest = fq[:, 2 * npairs:] @ fk[:, 2 * npairs:].T
    return rot + rest
