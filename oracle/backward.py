"""fp64 CPU oracle for the gradients of the hybrid attention forward (one batch element, one head).

TEST INFRASTRUCTURE ONLY, like the rest of `oracle/`: the library never imports it.

The backward pass is defined as the derivative of the forward pass, so the plainest correct statement
of it is the forward written with differentiable fp64 PyTorch CPU operations and differentiated by
autograd.  The block selection is piecewise constant in q and k (it only picks which key blocks each
query block attends to), so it is taken from the C oracle's forward and held fixed: gradients flow
through the attention over the kept blocks and through the low-rank branch, not through the choice of
blocks.

The restatement follows the forward's steps (RoLA "3 Preliminary" 3D RoPE, "4.1" block-sparse softmax
attention plus the low-rank branch, "4.2"/"4.3" rank-truncated RoPE outside the relu feature map,
"B.1" the query-independent summary):
  q^, k^ = RoPE(q), RoPE(k)                      (pairs (2j, 2j+1), the C oracle's own cos/sin)
  O_s    = softmax(q^ k^T / sqrt(D) over the kept key blocks of each query block) v
  phi    = relu(x A);  psi = phi with its first r coordinates rotated by the truncated RoPE
  S      = sum_j psi(k_j) v_j^T,  z = sum_j phi(k_j)
  O_lr   = psi(q) S / (phi(q) . z + 1e-6)
  out    = O_s + O_lr
The options of the forward are restated too: the feature map (relu, SiLU, identity, tanh), the
low-rank RoPE outside the activation, absent or inside it (psi = act(R x A), normaliser on psi), a
separate key projection, and the gated fusion of the two outputs.

The cos/sin of every (token, pair) come from the C oracle's rotation of unit vectors, so both
restatements use the same tables; `tests/test_oracle_pins.py` pins this forward to the C oracle's and
its gradients to finite differences and to torch's dense attention backward.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import ACT_IDENTITY, ACT_RELU, ACT_SILU, block_means, block_scores, keep_count, rope_rows, topk


def rope_cos_sin(grid, D: int, theta: float = 1e4, offset=(0, 0, 0), split=None) -> np.ndarray:
    """[L, D/2, 2] (cos, sin) of every token and rotary pair of a D-wide head: the C oracle's rotation
    applied to the unit vector of each pair's first coordinate."""
    T, H, W = grid
    L = T * H * W
    e = np.zeros((L, D))
    e[:, 0::2] = 1.0
    y = rope_rows(e, grid, D // 2, theta, offset, split)
    return np.stack([y[:, 0::2], y[:, 1::2]], axis=-1)


def _rotate(x: torch.Tensor, cs: torch.Tensor, npairs: int) -> torch.Tensor:
    """Rotate pairs (2j, 2j+1), j < npairs, of every row of x by the angles whose cos/sin are cs."""
    x0, x1 = x[:, 0:2 * npairs:2], x[:, 1:2 * npairs:2]
    c, s = cs[:, :npairs, 0], cs[:, :npairs, 1]
    y = x.clone()
    y[:, 0:2 * npairs:2] = x0 * c - x1 * s
    y[:, 1:2 * npairs:2] = x0 * s + x1 * c
    return y


def block_mask(idx: np.ndarray, L: int, block: int) -> torch.Tensor:
    """[L, L] bool: query i may attend key j iff j's block is kept for i's block."""
    nb = idx.shape[0]
    kept = np.zeros((nb, nb), dtype=bool)
    for a in range(nb):
        kept[a, idx[a]] = True
    bl = np.arange(L) // block
    return torch.from_numpy(kept[bl][:, bl])


def _act(u: torch.Tensor, act: int) -> torch.Tensor:
    if act == ACT_RELU:
        return torch.relu(u)
    if act == ACT_SILU:
        return u / (1.0 + torch.exp(-u))
    if act == ACT_IDENTITY:
        return u
    return torch.tanh(u)


def forward_torch(q, k, v, A, cs, mask, rank: int, branches: int = 3, *, activation: int = ACT_RELU,
                  rope: str = "outside", A_k=None, gate=None) -> torch.Tensor:
    """The forward of one head in differentiable fp64 torch (see the module docstring).  rope is
    "outside", "none" or "inside"; A_k a separate key projection; gate = (w, b) tensors."""
    L, D = q.shape
    o_s = torch.zeros_like(v)
    if branches & 1:
        qh, kh = _rotate(q, cs, D // 2), _rotate(k, cs, D // 2)
        s = (qh @ kh.T) / math.sqrt(D)
        s = s.masked_fill(~mask, float("-inf"))
        o_s = torch.softmax(s, dim=1) @ v
    if not branches & 2:
        return o_s
    Ak = A if A_k is None else A_k
    if rope == "inside":
        psq = _act(_rotate(q @ A, cs, rank // 2), activation)
        psk = _act(_rotate(k @ Ak, cs, rank // 2), activation)
        phq, phk = psq, psk
    else:
        phq, phk = _act(q @ A, activation), _act(k @ Ak, activation)
        if rope == "outside":
            psq, psk = _rotate(phq, cs, rank // 2), _rotate(phk, cs, rank // 2)
        else:
            psq, psk = phq, phk
    S, z = psk.T @ v, phk.sum(0)
    o_lr = (psq @ S) / (phq @ z + 1e-6)[:, None]
    if gate is None:
        return o_s + o_lr
    w, b = gate
    g = torch.sigmoid(q @ w + b)[:, None]
    rms_s = torch.sqrt((o_s * o_s).mean(1, keepdim=True))
    rms_l = torch.sqrt((o_lr * o_lr).mean(1, keepdim=True) + 1e-6)
    return o_s + g * o_lr * rms_s / rms_l


def head_backward(q, k, v, A, dout, grid, block: int, keep_frac: float, rank: int, *, theta=1e4,
                  offset=(0, 0, 0), split=None, branches: int = 3, idx=None, activation: int = ACT_RELU,
                  rope: str = "outside", A_k=None, gate=None):
    """Gradients of sum(dout * out) with respect to q, k, v [L, D], A [D, R] and (when given) the key
    projection A_k and the gate weights and bias (all fp64 numpy), the block selection held at the
    forward's (or `idx`).  Returns dict(dq, dk, dv, dA, [dA_k], [dgate_w, dgate_b], out, idx)."""
    L, D = q.shape
    if idx is None:
        qh = rope_rows(q, grid, D // 2, theta, offset, split)
        kh = rope_rows(k, grid, D // 2, theta, offset, split)
        s = block_scores(block_means(qh, block), block_means(kh, block))
        idx, _ = topk(s, keep_count(keep_frac, s.shape[0]))
    cs = torch.from_numpy(rope_cos_sin(grid, D, theta, offset, split))
    mask = block_mask(np.asarray(idx), L, block)
    leaf = lambda a: torch.tensor(np.asarray(a, dtype=np.float64), requires_grad=True)
    tq, tk, tv, tA = (leaf(a) for a in (q, k, v, A))
    extra, names = [], []
    tAk = None
    if A_k is not None:
        tAk = leaf(A_k)
        extra.append(tAk)
        names.append("dA_k")
    tgate = None
    if gate is not None:
        tgate = (leaf(gate[0]), leaf(float(gate[1])))
        extra += list(tgate)
        names += ["dgate_w", "dgate_b"]
    out = forward_torch(tq, tk, tv, tA, cs, mask, rank, branches, activation=activation, rope=rope, A_k=tAk,
                        gate=tgate)
    grads = torch.autograd.grad(out, [tq, tk, tv, tA] + extra,
                                torch.from_numpy(np.asarray(dout, dtype=np.float64)), allow_unused=True)
    refs = [q, k, v, A] + [a.detach().numpy() for a in extra]
    z = lambda g, ref: np.zeros_like(np.asarray(ref, dtype=np.float64)) if g is None else g.numpy()
    res = dict(zip(["dq", "dk", "dv", "dA"] + names, (z(g, r) for g, r in zip(grads, refs))))
    res.update(out=out.detach().numpy(), idx=np.asarray(idx))
    return res


def _unrotate(y: np.ndarray, cs: np.ndarray, npairs: int) -> np.ndarray:
    """R(p)^T y: rotate pairs (2j, 2j+1), j < npairs, back by their angles."""
    x = y.copy()
    c, s = cs[:, :npairs, 0], cs[:, :npairs, 1]
    y0, y1 = y[:, 0:2 * npairs:2], y[:, 1:2 * npairs:2]
    x[:, 0:2 * npairs:2] = y0 * c + y1 * s
    x[:, 1:2 * npairs:2] = -y0 * s + y1 * c
    return x


def _rot_np(x: np.ndarray, cs: np.ndarray, npairs: int) -> np.ndarray:
    y = x.copy()
    c, s = cs[:, :npairs, 0], cs[:, :npairs, 1]
    x0, x1 = x[:, 0:2 * npairs:2], x[:, 1:2 * npairs:2]
    y[:, 0:2 * npairs:2] = x0 * c - x1 * s
    y[:, 1:2 * npairs:2] = x0 * s + x1 * c
    return y


def head_backward_steps(q, k, v, A, dout, grid, block: int, rank: int, idx, *, theta=1e4, offset=(0, 0, 0),
                        split=None):
    """The same gradients as head_backward (relu features, RoPE outside, one shared projection, plain
    sum), written as the explicit steps a kernel takes, in fp64 numpy:

    sparse branch (per query row i over its allowed keys j):
      s_ij = q^_i . k^_j / sqrt(D),  lse_i = log sum_j exp(s_ij),  P_ij = exp(s_ij - lse_i)
      Delta_i = dO_i . O_s,i,  dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - Delta_i)
      dq^_i = sum_j dS_ij k^_j / sqrt(D),  dk^_j = sum_i dS_ij q^_i / sqrt(D),  dv_j += sum_i P_ij dO_i
      dq += R(p_i)^T dq^_i,  dk += R(p_j)^T dk^_j
    low-rank branch (u = x A, phi = relu(u), psi = R_r phi, den_i = phi_q,i . z + 1e-6):
      dpsi_q,i = S dO_i / den_i,  dden_i = -(dO_i . O_lr,i) / den_i,  dphi_q,i = R_r^T dpsi_q,i + dden_i z
      dS = sum_i psi_q,i dO_i^T / den_i,  dz = sum_i dden_i phi_q,i
      dpsi_k,j = dS v_j,  dv_j += dS^T psi_k,j,  dphi_k,j = R_r^T dpsi_k,j + dz
      du = dphi * [u > 0],  dq += du_q A^T,  dk += du_k A^T,  dA = q^T du_q + k^T du_k
    Returns dict(dq, dk, dv, dA)."""
    q, k, v, A, dout = (np.asarray(a, dtype=np.float64) for a in (q, k, v, A, dout))
    L, D = q.shape
    cs = rope_cos_sin(grid, D, theta, offset, split)
    mask = block_mask(np.asarray(idx), L, block).numpy()
    # sparse branch
    qh, kh = _rot_np(q, cs, D // 2), _rot_np(k, cs, D // 2)
    s = np.where(mask, qh @ kh.T / math.sqrt(D), -np.inf)
    m = s.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(s - m).sum(axis=1, keepdims=True))
    P = np.exp(s - lse)
    o_s = P @ v
    delta = (dout * o_s).sum(axis=1, keepdims=True)
    dS = P * (dout @ v.T - delta)
    dqh, dkh = dS @ kh / math.sqrt(D), dS.T @ qh / math.sqrt(D)
    dv = P.T @ dout
    dq, dk = _unrotate(dqh, cs, D // 2), _unrotate(dkh, cs, D // 2)
    # low-rank branch
    r2 = rank // 2
    uq, uk = q @ A, k @ A
    phq, phk = np.maximum(uq, 0.0), np.maximum(uk, 0.0)
    psq, psk = _rot_np(phq, cs, r2), _rot_np(phk, cs, r2)
    Sm, z = psk.T @ v, phk.sum(axis=0)
    den = phq @ z + 1e-6
    o_lr = (psq @ Sm) / den[:, None]
    dpsq = (dout @ Sm.T) / den[:, None]
    dden = -(dout * o_lr).sum(axis=1) / den
    dphq = _unrotate(dpsq, cs, r2) + dden[:, None] * z[None, :]
    dSm = psq.T @ (dout / den[:, None])
    dz = dden @ phq
    dpsk = v @ dSm.T
    dv = dv + psk @ dSm
    dphk = _unrotate(dpsk, cs, r2) + dz[None, :]
    duq, duk = dphq * (uq > 0), dphk * (uk > 0)
    dq = dq + duq @ A.T
    dk = dk + duk @ A.T
    dA = q.T @ duq + k.T @ duk
    return dict(dq=dq, dk=dk, dv=dv, dA=dA)


def head_backward_sampled(q, k, v, A, dout, grid, block: int, rank: int, idx, qblocks, kblocks, *, theta=1e4,
                          offset=(0, 0, 0), split=None):
    """The gradients of head_backward_steps (relu features, RoPE outside, one shared projection, plain
    sum) evaluated only where asked: dq on the rows of the query blocks `qblocks`, dk and dv on the rows
    of the key blocks `kblocks`, and dA in full.  The sparse terms of a query row involve only its own
    kept key blocks; those of a key row involve only the query blocks that kept its block (each with its
    own softmax over its own kept set); the low-rank terms need the global sums S, z, dS, dz, which are
    O(L r D).  So a full-size head is affordable in fp64.  Returns dict(dq={alpha: [rows, D]},
    dk={beta: [rows, D]}, dv={beta: [rows, D]}, dA)."""
    q, k, v, A, dout = (np.asarray(a, dtype=np.float64) for a in (q, k, v, A, dout))
    L, D = q.shape
    nb = idx.shape[0]
    cs = rope_cos_sin(grid, D, theta, offset, split)
    sc = 1.0 / math.sqrt(D)
    qh, kh = _rot_np(q, cs, D // 2), _rot_np(k, cs, D // 2)
    rows = lambda a: np.arange(a * block, min(L, (a + 1) * block))
    keys = lambda a: np.concatenate([rows(b) for b in idx[a]])

    def softmax_block(a):
        """P, dS over the kept keys of query block a (rows of a x kept keys), and those keys."""
        r, kk = rows(a), keys(a)
        s = qh[r] @ kh[kk].T * sc
        s = s - s.max(axis=1, keepdims=True)
        P = np.exp(s)
        P /= P.sum(axis=1, keepdims=True)
        o_s = P @ v[kk]
        delta = (dout[r] * o_s).sum(axis=1, keepdims=True)
        dS = P * (dout[r] @ v[kk].T - delta)
        return r, kk, P, dS

    # low-rank branch: global sums
    r2 = rank // 2
    uq, uk = q @ A, k @ A
    phq, phk = np.maximum(uq, 0.0), np.maximum(uk, 0.0)
    psq, psk = _rot_np(phq, cs, r2), _rot_np(phk, cs, r2)
    Sm, z = psk.T @ v, phk.sum(axis=0)
    den = phq @ z + 1e-6
    G = dout @ Sm.T
    dden = -(psq * G).sum(axis=1) / den ** 2
    dphq = _unrotate(G / den[:, None], cs, r2) + dden[:, None] * z[None, :]
    dSm = psq.T @ (dout / den[:, None])
    dz = dden @ phq
    dphk = _unrotate(v @ dSm.T, cs, r2) + dz[None, :]
    duq, duk = dphq * (uq > 0), dphk * (uk > 0)
    dA = q.T @ duq + k.T @ duk
    out = dict(dq={}, dk={}, dv={}, dA=dA)
    for a in qblocks:
        r, kk, P, dS = softmax_block(a)
        dqh = dS @ kh[kk] * sc
        out["dq"][a] = _unrotate(dqh, cs[r], D // 2) + duq[r] @ A.T
    for b in kblocks:
        kr = rows(b)
        dkh = np.zeros((kr.size, D))
        dvs = np.zeros((kr.size, D))
        for a in range(nb):
            if b not in idx[a]:
                continue
            r, kk, P, dS = softmax_block(a)
            pos = np.searchsorted(kk, kr) if np.all(np.diff(kk) > 0) else None
            sel = pos if pos is not None else np.array([np.where(kk == j)[0][0] for j in kr])
            dvs += P[:, sel].T @ dout[r]
            dkh += dS[:, sel].T @ qh[r] * sc
        out["dk"][b] = _unrotate(dkh, cs[kr], D // 2) + duk[kr] @ A.T
        out["dv"][b] = dvs + psk[kr] @ dSm
    return out
