"""fp64 CPU oracle for 3D-RoPE sparse + low-rank hybrid attention (forward pass).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg use this
package; the library (`sparse_rank_hybrid_b200`) never imports it, and it imports nothing from the
library.  The arithmetic lives in `slra_oracle.c` (plain fp64 loops); this module only decodes the
bf16 inputs, slices one (batch, head) at a time and strings the steps together in the order the
method defines them:

  1. 3D RoPE on q and k (RoLA, "3 Preliminary"; rotary base 10000, head split over t/h/w).
  2. Block mean pooling of the rotated q and k, block scores qbar . kbar.
  3. Per query block, top-k key blocks by (score desc, block index asc) plus a tie flag.
  4. Block-sparse softmax attention over the kept blocks (RoLA "4.1").
  5. Low-rank branch: phi = relu(x A) on raw q/k, rank-truncated RoPE outside the activation
     (RoLA "4.2", "4.3"), summary S = sum_j psi(k_j) v_j^T and z = sum_j phi(k_j) once per head
     ("B.1"), readout psi(q_i)^T S / (phi(q_i) . z + 1e-6).
  6. out = sparse branch + low-rank branch.

Parity status per function is stated in the tests that pin it; the absolute output values have no
worked example on the pages, so they are pinned only through the properties and special cases
listed there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "slra_oracle.c")
_LIB = os.path.join(_HERE, "libslra_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, OpenMP, no fast-math) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        _lib.orc_keep_count.restype = ctypes.c_int64
        _lib.orc_keep_count.argtypes = [ctypes.c_double, I]
        _lib.orc_rope_pairs.restype = ctypes.c_int
        _lib.orc_rope_pairs.argtypes = [I, P, ctypes.c_double, P, P]
        _lib.orc_decode_bf16.argtypes = [P, I, P]
        _lib.orc_rope_rows.argtypes = [P, I, I, I, I, I, P, P, P, I, P]
        _lib.orc_block_means.argtypes = [P, I, I, I, P]
        _lib.orc_block_scores.argtypes = [P, P, I, I, P]
        _lib.orc_topk.argtypes = [P, I, I, P, P]
        _lib.orc_sparse_attn.argtypes = [P, P, P, I, I, I, P, I, P, I, P]
        _lib.orc_features.argtypes = [P, I, I, P, I, ctypes.c_int, P]
        _lib.orc_summary.argtypes = [P, P, P, I, I, I, P, P]
        _lib.orc_lowrank_apply.argtypes = [P, P, P, P, I, I, P, I, P]
        _lib.orc_gated_fusion.argtypes = [P, P, P, P, ctypes.c_double, I, P, I, P]
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().orc_decode_bf16(_p(bits), bits.size, _p(out))
    return out


def keep_count(keep_frac: float, nb: int) -> int:
    return int(_load().orc_keep_count(float(keep_frac), int(nb)))


def rope_pairs(D: int, theta: float = 1e4, split=None):
    """(axis[j], omega[j]) for the D/2 rotary pairs; split = pairs per (t, h, w) or None (default)."""
    axis = np.empty(D // 2, dtype=np.int32)
    omega = np.empty(D // 2, dtype=np.float64)
    sp = None if split is None else np.ascontiguousarray(split, dtype=np.int64)
    rc = _load().orc_rope_pairs(D, None if sp is None else _p(sp), float(theta), _p(axis), _p(omega))
    if rc != 0:
        raise ValueError(f"bad rope split {split} for D={D}")
    return axis, omega


def rope_rows(x: np.ndarray, grid, npairs: int, theta: float = 1e4, offset=(0, 0, 0), split=None,
              schedule_dim: int | None = None) -> np.ndarray:
    """Rotate the first `npairs` pairs of every row of x [L, width] (fp64) at its grid position.

    The rotary schedule (axis and frequency of each pair) is that of a head of width
    `schedule_dim` (default: the row width).  The low-rank branch rotates R-wide feature rows with the
    first R/2 pairs of the D-wide schedule (RoLA "4.2": the first r rotary coordinates, reusing the
    backbone's cos/sin tensors), so it passes schedule_dim = D.
    """
    T, H, W = grid
    x = np.ascontiguousarray(x, dtype=np.float64)
    L, width = x.shape
    axis, omega = rope_pairs(width if schedule_dim is None else schedule_dim, theta, split)
    assert npairs <= axis.size and 2 * npairs <= width
    off = np.ascontiguousarray(offset, dtype=np.int64)
    y = np.empty_like(x)
    _load().orc_rope_rows(_p(x), L, width, T, H, W, _p(off), _p(axis), _p(omega), int(npairs), _p(y))
    return y


def block_means(x: np.ndarray, block: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    L, D = x.shape
    nb = -(-L // block)
    out = np.empty((nb, D), dtype=np.float64)
    _load().orc_block_means(_p(x), L, D, block, _p(out))
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    nb, D = qbar.shape
    s = np.empty((nb, nb), dtype=np.float64)
    _load().orc_block_scores(_p(qbar), _p(kbar), nb, D, _p(s))
    return s


def topk(s: np.ndarray, k: int):
    s = np.ascontiguousarray(s, dtype=np.float64)
    nb = s.shape[0]
    idx = np.empty((nb, k), dtype=np.int32)
    tie = np.empty(nb, dtype=np.uint8)
    _load().orc_topk(_p(s), nb, k, _p(idx), _p(tie))
    return idx, tie


def sparse_attn(qh, kh, v, block: int, idx: np.ndarray, qblocks=None) -> np.ndarray:
    qh = np.ascontiguousarray(qh, dtype=np.float64)
    kh = np.ascontiguousarray(kh, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    L, D = qh.shape
    nb, k = idx.shape
    qb = np.arange(nb, dtype=np.int64) if qblocks is None else np.ascontiguousarray(qblocks, dtype=np.int64)
    out = np.full((L, D), np.nan)
    _load().orc_sparse_attn(_p(qh), _p(kh), _p(v), L, D, block, _p(idx), k, _p(qb), qb.size, _p(out))
    return out


ACT_RELU, ACT_SILU, ACT_IDENTITY, ACT_TANH = 0, 1, 2, 3


def features(x: np.ndarray, A: np.ndarray, act: int = ACT_RELU) -> np.ndarray:
    """phi = act(x A): relu (default), SiLU, identity or tanh (RoLA 5.3, Table 6)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    A = np.ascontiguousarray(A, dtype=np.float64)
    L, D = x.shape
    R = A.shape[1]
    phi = np.empty((L, R), dtype=np.float64)
    _load().orc_features(_p(x), L, D, _p(A), R, int(act), _p(phi))
    return phi


def summary(psik, phik, v):
    psik = np.ascontiguousarray(psik, dtype=np.float64)
    phik = np.ascontiguousarray(phik, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    L, R = psik.shape
    D = v.shape[1]
    S = np.empty((R, D), dtype=np.float64)
    z = np.empty(R, dtype=np.float64)
    _load().orc_summary(_p(psik), _p(phik), _p(v), L, R, D, _p(S), _p(z))
    return S, z


def lowrank_apply(psiq, phiq, S, z, rows=None) -> np.ndarray:
    psiq = np.ascontiguousarray(psiq, dtype=np.float64)
    phiq = np.ascontiguousarray(phiq, dtype=np.float64)
    S = np.ascontiguousarray(S, dtype=np.float64)
    z = np.ascontiguousarray(z, dtype=np.float64)
    L, R = psiq.shape
    D = S.shape[1]
    rr = np.arange(L, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.full((L, D), np.nan)
    _load().orc_lowrank_apply(_p(psiq), _p(phiq), _p(S), _p(z), R, D, _p(rr), rr.size, _p(out))
    return out


def gated_fusion(o_s, o_lr, q, w, b: float, rows) -> np.ndarray:
    """out_i = O_s,i + sigmoid(q_i . w + b) * O_lr,i * rms(O_s,i) / sqrt(mean(O_lr,i^2) + 1e-6) for the
    given rows (RoLA 4.4's token-wise gate with the sparse output's RMS as scale reference; the
    formula is this implementation's reading, see slra_oracle.c)."""
    o_s, o_lr, q = (np.ascontiguousarray(a, dtype=np.float64) for a in (o_s, o_lr, q))
    w = np.ascontiguousarray(w, dtype=np.float64)
    L, D = o_s.shape
    rr = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((L, D))
    _load().orc_gated_fusion(_p(o_s), _p(o_lr), _p(q), _p(w), float(b), D, _p(rr), rr.size, _p(out))
    return out


def head_forward(q, k, v, A, grid, block: int, keep_frac: float, rank: int, *, theta=1e4,
                 offset=(0, 0, 0), split=None, qblocks=None, branches=3, idx_override=None,
                 activation=ACT_RELU, lowrank_rope=True, A_k=None, gate=None, rope_inside=False):
    """Forward pass of one (batch, head): q, k, v fp64 [L, D]; A fp64 [D, R].

    `activation` picks the feature map's nonlinearity; `lowrank_rope=False` drops the truncated RoPE
    from the low-rank branch (psi = phi), the no-RoPE setting of RoLA's ablation (5.3).  `A_k`, when
    given, is a separate key projection Pk (RoLA E.2 lists Pq and Pk as the branch's parameters):
    query features use A, key features use A_k.  `rope_inside=True` applies the truncated RoPE to the
    projected features BEFORE the activation, psi = act(R_r(p) x A), the ordering RoLA's ablation
    compares against (5.1 Table 2, 5.3, B.3); numerator and normaliser then both use psi (there is no
    unrotated feature left to normalise with), so the summary stays linear but loses the relative
    property.  `gate=(w, b)` replaces the plain sum of the two
    branches by the gated fusion of RoLA 4.4 (see gated_fusion; needs both branches).

    Returns a dict with out (rows of the computed query blocks; NaN elsewhere), the sparse and
    low-rank branch outputs, the rotated q/k, block means, scores, idx, tie flags, S and z.
    `idx_override` replaces the oracle's own top-k selection (used to compare a tie-flagged row
    under another implementation's equally valid mask).
    """
    L, D = q.shape
    R = rank
    qh = rope_rows(q, grid, D // 2, theta, offset, split)
    kh = rope_rows(k, grid, D // 2, theta, offset, split)
    qbar = block_means(qh, block)
    kbar = block_means(kh, block)
    s = block_scores(qbar, kbar)
    nb = s.shape[0]
    kk = keep_count(keep_frac, nb)
    idx, tie = topk(s, kk)
    use_idx = idx if idx_override is None else np.ascontiguousarray(idx_override, dtype=np.int32)
    qb = np.arange(nb, dtype=np.int64) if qblocks is None else np.asarray(qblocks, dtype=np.int64)
    rows = np.concatenate([np.arange(a * block, min(L, (a + 1) * block)) for a in qb]) if qb.size else \
        np.zeros(0, dtype=np.int64)
    res = dict(qh=qh, kh=kh, qbar=qbar, kbar=kbar, scores=s, idx=idx, tie=tie, keep=kk)
    out = np.zeros((L, D))
    out[:] = np.nan
    out[rows] = 0.0
    if branches & 1:
        o_s = sparse_attn(qh, kh, v, block, use_idx, qb)
        res["out_sparse"] = o_s
        out[rows] += o_s[rows]
    if rope_inside:
        assert lowrank_rope, "RoPE inside the activation needs the low-rank RoPE"
        Ak = A if A_k is None else A_k
        yq = rope_rows(features(q, A, ACT_IDENTITY), grid, R // 2, theta, offset, split, schedule_dim=D)
        yk = rope_rows(features(k, Ak, ACT_IDENTITY), grid, R // 2, theta, offset, split, schedule_dim=D)
        eye = np.eye(R)  # act(y I) = act(y) exactly in fp64
        psiq, psik = features(yq, eye, activation), features(yk, eye, activation)
        phiq, phik = psiq, psik
    else:
        phiq = features(q, A, activation)
        phik = features(k, A if A_k is None else A_k, activation)
        if lowrank_rope:
            psiq = rope_rows(phiq, grid, R // 2, theta, offset, split, schedule_dim=D)
            psik = rope_rows(phik, grid, R // 2, theta, offset, split, schedule_dim=D)
        else:
            psiq, psik = phiq.copy(), phik.copy()
    S, z = summary(psik, phik, v)
    res.update(S=S, z=z, phiq=phiq, phik=phik, psiq=psiq, psik=psik)
    if branches & 2:
        o_lr = lowrank_apply(psiq, phiq, S, z, rows)
        res["out_lowrank"] = o_lr
        if gate is None:
            out[rows] += o_lr[rows]
        else:
            assert branches == 3, "the gated fusion combines both branches"
            out[rows] = gated_fusion(res["out_sparse"], o_lr, q, gate[0], gate[1], rows)[rows]
    res["out"] = out
    return res


def forward(inp: dict, grid, block: int, keep_frac: float, rank: int, *, theta=1e4, offset=(0, 0, 0),
            split=None, heads=None, qblocks=None, branches=3, idx_override=None, keep_intermediates=False,
            activation=ACT_RELU, lowrank_rope=True, proj_separate=False, proj_per_head=False, gate=None,
            rope_inside=False):
    """Full forward over all (batch, head) pairs of bf16 inputs q, k, v [B, L, Hh, D] and A [D, R].

    With `proj_separate` and/or `proj_per_head`, A holds [1 + separate][per_head ? Hh : 1][D][R]
    bf16 values: the query projection(s) first, then the key projection(s) (RoLA E.2's Pq, Pk;
    RoPeSLR's head-wise low-rank parameterization); head h uses entry h of each.  `gate=(w, b)`: the
    gated fusion of the branches (w fp64 [D] shared by all heads, b a scalar).

    heads: optional list of (b, h) to compute (default all).  qblocks: dict {(b, h): [alpha...]} or a
    list applied to every head (default all query blocks).  Returns per-(b, h) dicts of results plus
    the assembled output `out` [B, L, Hh, D] (NaN where not computed).
    """
    q, k, v, A = inp["q"], inp["k"], inp["v"], inp["A"]
    B, L, Hh, D = q.shape
    Af = decode_bf16(A).reshape(2 if proj_separate else 1, Hh if proj_per_head else 1, D, rank)
    pairs = [(b, h) for b in range(B) for h in range(Hh)] if heads is None else list(heads)
    out = np.full((B, L, Hh, D), np.nan)
    per = {}
    for (b, h) in pairs:
        qb = qblocks.get((b, h), []) if isinstance(qblocks, dict) else qblocks
        ov = None if idx_override is None else idx_override[b, h]
        r = head_forward(decode_bf16(q[b, :, h, :]), decode_bf16(k[b, :, h, :]), decode_bf16(v[b, :, h, :]),
                         Af[0, h if proj_per_head else 0], grid, block, keep_frac, rank, theta=theta,
                         offset=offset, split=split, qblocks=qb, branches=branches, idx_override=ov,
                         activation=activation, lowrank_rope=lowrank_rope,
                         A_k=Af[-1, h if proj_per_head else 0], gate=gate, rope_inside=rope_inside)
        out[b, :, h, :] = r["out"]
        if not keep_intermediates:
            for key in ("qh", "kh", "phiq", "phik", "psiq", "psik", "out_sparse", "out_lowrank", "out"):
                r.pop(key, None)
        per[(b, h)] = r
    return out, per
