"""Shared helpers for the GPU parity tests: move seeded inputs to the GPU, run the C-ABI path,
compute the oracle on the same bytes, and compare with the acceptance tolerances.

Tolerances (stated once, used by every parity test): block masks bit-exact except rows whose
selection is within the tie band (any set valid under the oracle's scores is accepted there);
outputs within max-abs error 1e-2 and mean relative error sum|o - o*| / sum|o*| <= 2e-3 of the fp64
oracle; the low-rank summary S, z within 1e-4 relative Frobenius norm (fp32 accumulation over L keys).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_rank_hybrid_b200 import slra

MAX_ABS = 1e-2
MEAN_REL = 2e-3
SUMMARY_REL = 1e-4


def to_gpu(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_gpu(prob: slra.Problem, x: dict, expect_status: int = slra.OK):
    q, k, v, A = (to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    out, ws = slra.attn_fwd(prob, q, k, v, A)
    st = slra.device_status(ws)
    assert st == expect_status, slra.status_string(st)
    res = {"out": out.float().cpu().numpy().astype(np.float64)}
    if prob.branches & slra.BRANCH_SPARSE:
        res["idx"] = slra.ws_view(prob, ws, "idx").cpu().numpy()
        res["tie"] = slra.ws_view(prob, ws, "tie").cpu().numpy()
        res["qbar"] = slra.ws_view(prob, ws, "qbar").cpu().numpy()
        res["kbar"] = slra.ws_view(prob, ws, "kbar").cpu().numpy()
    if prob.branches & slra.BRANCH_LOWRANK:
        res["S"] = slra.ws_view(prob, ws, "S").cpu().numpy().astype(np.float64)
        res["z"] = slra.ws_view(prob, ws, "z").cpu().numpy().astype(np.float64)
    return res


def mask_ok(idx_gpu: np.ndarray, s_orc: np.ndarray, idx_orc: np.ndarray, tie_orc: np.ndarray, keep: int):
    """Per row: True if the GPU's kept set equals the oracle's, or (tie-band row) is a valid top-k
    under the oracle's scores within the band.  Returns (all_ok, rows_differing)."""
    nb = s_orc.shape[0]
    diff = []
    for a in range(nb):
        g = np.sort(idx_gpu[a])
        if np.array_equal(g, idx_orc[a]):
            continue
        diff.append(a)
        srt = np.sort(s_orc[a])[::-1]
        sk = srt[keep - 1]
        band = 1e-6 * max(1.0, abs(sk))
        sel = np.zeros(nb, bool)
        sel[g] = True
        if len(set(g.tolist())) != keep:
            return False, diff
        if not (np.all(s_orc[a][~sel] <= sk + band) and np.all(s_orc[a][sel] >= sk - band)):
            return False, diff
    return True, diff


def _gate_of(prob: slra.Problem):
    """The oracle's gate argument for a gated problem: (Wg as fp64, bg rounded to fp32 as the library
    receives it), else None."""
    if prob.fusion != slra.FUSION_GATED:
        return None
    return prob.gate_w.detach().cpu().numpy().astype(np.float64), float(np.float32(prob.gate_bias))


def compare(prob: slra.Problem, x: dict, gpu: dict, heads=None, qblocks=None, check_masks=True, label="",
            max_abs: float = MAX_ABS):
    """Run the oracle on (a sample of) the problem and compare.  Returns a dict of error stats.
    `max_abs` replaces the absolute bound for inputs whose v is scaled by s (the output scales with v,
    so the same accuracy is 1e-2 * s there); the mean relative bound never changes."""
    grid = (prob.T, prob.H, prob.W)
    B, Hh = prob.batch, prob.heads
    pairs = [(b, h) for b in range(B) for h in range(Hh)] if heads is None else heads
    override = None
    if "idx" in gpu:
        override = gpu["idx"].reshape(B, Hh, *gpu["idx"].shape[1:])
    out_o, per = oracle.forward(x, grid, prob.block, prob.keep_frac, prob.rank, offset=prob.pos_offset,
                                heads=pairs, qblocks=qblocks, branches=prob.branches, idx_override=override,
                                activation=prob.activation, lowrank_rope=not prob.lowrank_norope,
                                proj_separate=bool(prob.proj_separate), proj_per_head=bool(prob.proj_per_head),
                                gate=_gate_of(prob), rope_inside=bool(prob.lowrank_rope_inside))
    stats = {"label": label, "mask_rows_differing": 0, "mask_rows": 0}
    for (b, h) in pairs:
        r = per[(b, h)]
        bh = b * Hh + h
        if "idx" in gpu and check_masks:
            ok, diff = mask_ok(gpu["idx"][bh], r["scores"], r["idx"], r["tie"], r["keep"])
            assert ok, f"{label}: mask mismatch outside the tie band at (b={b}, h={h}) rows {diff[:8]}"
            stats["mask_rows_differing"] += len(diff)
            stats["mask_rows"] += r["idx"].shape[0]
            # rows not tie-flagged must agree exactly
            assert all(r["tie"][a] or gpu["tie"][bh][a] for a in diff), f"{label}: untied row differs"
            qb_err = np.abs(gpu["qbar"][bh] - r["qbar"]).max() / max(1e-300, np.abs(r["qbar"]).max())
            stats["qbar_rel"] = max(stats.get("qbar_rel", 0.0), qb_err)
            assert qb_err < 1e-12, f"{label}: block means differ {qb_err}"
        if "S" in gpu:
            es = np.linalg.norm(gpu["S"][bh] - r["S"]) / max(1e-300, np.linalg.norm(r["S"]))
            ez = np.linalg.norm(gpu["z"][bh] - r["z"]) / max(1e-300, np.linalg.norm(r["z"]))
            stats["S_rel"] = max(stats.get("S_rel", 0.0), es)
            stats["z_rel"] = max(stats.get("z_rel", 0.0), ez)
            assert es < SUMMARY_REL and ez < SUMMARY_REL, f"{label}: summary S {es:.3g} z {ez:.3g}"
    sel = ~np.isnan(out_o)
    assert sel.any()
    o, g = out_o[sel], gpu["out"][sel]
    assert np.all(np.isfinite(g)), f"{label}: non-finite GPU output"
    err = np.abs(g - o)
    stats["max_abs"] = float(err.max())
    stats["mean_rel"] = float(err.sum() / np.abs(o).sum())
    stats["n_compared"] = int(sel.sum())
    assert stats["max_abs"] <= max_abs, f"{label}: max abs error {stats['max_abs']:.3g}"
    assert stats["mean_rel"] <= MEAN_REL, f"{label}: mean rel error {stats['mean_rel']:.3g}"
    return stats
