"""GPU parity of the backward pass (slra_attn_bwd) against the fp64 oracle's gradients.

The oracle is oracle/backward.py's head_backward: the forward restated in differentiable fp64 torch and
differentiated by autograd, pinned on the CPU to finite differences of the C oracle, to torch's dense
attention backward and to the explicit gradient steps.  Both sides use the same block selection (the
GPU's, read back from the workspace; the selection is piecewise constant, so gradients do not flow
through it).  dA is the sum over all heads and batch elements of the per-head gradients (A is shared).

Tolerance, derived from the arithmetic: the gradients go through fp16 operands (q^, k^, v, dO, P, dS;
2^-12 relative rounding each, the inputs exact in bf16) with fp32 accumulation, the same class of error
as the forward, whose mean relative error is ~3e-4 against a 2e-3 bound.  So every gradient tensor must
have mean relative error sum|g - g*| / sum|g*| <= 2e-3, and max-abs error <= 1e-2 * max|g*| (the
forward's absolute 1e-2 bound, scaled to the gradient's own magnitude, which grows with L and dout).
"""
import json
import os

import numpy as np
import pytest

from sparse_rank_hybrid_b200 import inputs as I
from sparse_rank_hybrid_b200 import slra
from sparse_rank_hybrid_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

MEAN_REL = 2e-3
MAX_ABS_REL = 1e-2
REPORT = os.environ.get("SLRA_PARITY_REPORT")


@pytest.fixture(scope="module", autouse=True)
def _build():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_rank_hybrid_b200 import build
    build.build()
    import oracle
    oracle.build()


def _gpu_bwd(w, x, dout, **kw):
    import torch
    p = slra.Problem.from_workload(w, **kw)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    g = torch.from_numpy(dout).cuda()
    dq, dk, dv, dA, ws = slra.attn_bwd(p, q, k, v, A, g)
    assert slra.device_status(ws) == slra.OK
    idx = slra.ws_view(p, ws, "idx").cpu().numpy() if p.branches & slra.BRANCH_SPARSE else None
    return p, [t.cpu().numpy().astype(np.float64) for t in (dq, dk, dv, dA)], idx


def _oracle_bwd(w, x, dout, idx, branches, activation=slra.ACT_RELU, rope="outside", separate=0, per_head=0):
    """The oracle's gradients head by head; dA in the projection argument's layout (query projections
    first, then the key projections when separate; one per head when per head)."""
    import oracle
    from oracle import backward as OB
    B, L, Hh, D = x["q"].shape
    R = w.rank
    nh = Hh if per_head else 1
    P = oracle.decode_bf16(x["A"]).reshape(1 + separate, nh, D, R)
    grid = (w.T, w.H, w.W)
    ref = [np.zeros((B, L, Hh, D)) for _ in range(3)] + [np.zeros((1 + separate, nh, D, R))]
    for b in range(B):
        for h in range(Hh):
            hidx = None if idx is None else idx[b * Hh + h]
            if hidx is None:  # low-rank only: any selection (unused)
                hidx = np.zeros((w.nb, 1), dtype=np.int32)
            hp = h if per_head else 0
            r = OB.head_backward(oracle.decode_bf16(x["q"][b, :, h]), oracle.decode_bf16(x["k"][b, :, h]),
                                 oracle.decode_bf16(x["v"][b, :, h]), P[0, hp], dout[b, :, h].astype(np.float64),
                                 grid, w.block, w.keep_frac, R, branches=branches, idx=hidx, activation=activation,
                                 rope=rope, A_k=P[1, hp] if separate else None)
            ref[0][b, :, h] = r["dq"]
            ref[1][b, :, h] = r["dk"]
            ref[2][b, :, h] = r["dv"]
            ref[3][0, hp] += r["dA"]
            if separate:
                ref[3][1, hp] += r["dA_k"]
    if not separate and not per_head:
        ref[3] = ref[3].reshape(D, R)
    return ref


def _compare(label, got, ref):
    stats = {"label": label}
    for name, g, r in zip(("dq", "dk", "dv", "dA"), got, ref):
        assert np.all(np.isfinite(g)), f"{label}: non-finite {name}"
        err = np.abs(g - r)
        scale = np.abs(r).max()
        mean_rel = err.sum() / max(np.abs(r).sum(), 1e-300)
        stats[name] = {"max_abs": float(err.max()), "max_ref": float(scale), "mean_rel": float(mean_rel)}
        if scale == 0.0:
            assert err.max() == 0.0, f"{label}: {name} should be zero"
            continue
        assert err.max() <= MAX_ABS_REL * scale, f"{label}: {name} max abs {err.max():.3g} vs max {scale:.3g}"
        assert mean_rel <= MEAN_REL, f"{label}: {name} mean rel {mean_rel:.3g}"
    if REPORT:
        with open(REPORT, "a") as f:
            f.write(json.dumps(stats) + "\n")
    return stats


def _case(w, label, branches=slra.BRANCH_BOTH, dout_scale=1.0):
    x = I.make_inputs(w)
    dout = I.make_dout(w.seed + 9000, w.batch, w.L, w.heads, w.head_dim, dout_scale)
    p, got, idx = _gpu_bwd(w, x, dout, branches=branches)
    ref = _oracle_bwd(w, x, dout, idx, branches)
    return _compare(label, got, ref)


EDGE_128 = W.Workload("bwd-edge-128", 1, 2, 128, 3, 10, 13, 32, 128, 0.3, 7160)         # L = 390, ragged
EDGE_128_B64 = W.Workload("bwd-edge-128-b64", 1, 2, 128, 2, 9, 11, 64, 64, 0.25, 7192)  # block 64, r = 64
EDGE_B2 = W.Workload("bwd-edge-b2", 2, 3, 128, 2, 9, 11, 32, 64, 0.25, 7410)            # batch 2
DENSE = W.Workload("bwd-dense", 1, 2, 128, 4, 12, 16, 32, 128, 1.0, 7700)               # keep all
MEDIUM = W.Workload("bwd-medium", 1, 2, 128, 4, 24, 32, 32, 128, 0.1, 7800)             # L = 3072


@pytest.mark.parametrize("w", [W.TINY, EDGE_128, EDGE_128_B64, EDGE_B2, DENSE, MEDIUM], ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    _case(w, w.name)


@pytest.mark.parametrize("branches", [slra.BRANCH_SPARSE, slra.BRANCH_LOWRANK])
@pytest.mark.parametrize("w", [W.TINY, EDGE_128], ids=lambda w: w.name)
def test_backward_single_branch(w, branches):
    _case(w, f"{w.name}-branches{branches}", branches=branches)


def test_backward_deterministic_and_strided_inputs():
    """Two calls give the same bits, and q, k, v as views of one fused QKV buffer give the same bits."""
    import torch
    w = EDGE_128
    x = I.make_inputs(w)
    dout = torch.from_numpy(I.make_dout(1, w.batch, w.L, w.heads, w.head_dim)).cuda()
    p = slra.Problem.from_workload(w)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    a = slra.attn_bwd(p, q, k, v, A, dout)[:4]
    b = slra.attn_bwd(p, q, k, v, A, dout)[:4]
    qkv = torch.stack([q, k, v], dim=2).contiguous()
    c = slra.attn_bwd(p, qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], A, dout)[:4]
    for ta, tb, tc in zip(a, b, c):
        assert torch.equal(ta, tb) and torch.equal(ta, tc)


def test_backward_dout_range_reported():
    """A gradient too large for the fp16 operand copy is reported through the status word."""
    import torch
    w = W.TINY
    x = I.make_inputs(w)
    d = I.make_dout(2, w.batch, w.L, w.heads, w.head_dim)
    d[0, 3, 1, 5] = 1e6
    p = slra.Problem.from_workload(w)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    ws = slra.attn_bwd(p, q, k, v, A, torch.from_numpy(d).cuda())[4]
    assert slra.device_status(ws) == slra.ERR_RANGE


def test_backward_wan_1_3b_sampled():
    """The full Wan2.1-1.3B shape (32,760 tokens, 12 heads, keep 26/256): the GPU backward of the whole
    problem, compared on a sampled head's dq over sampled query blocks (first, last = ragged, random) and
    dk, dv over sampled key blocks (first, last, and the most-kept one), and dA (all heads) against the
    oracle's sampled gradients (head_backward_sampled, the explicit steps restricted to those rows)."""
    import oracle
    from oracle import backward as OB
    w = W.WAN_1_3B
    x = I.make_inputs(w)
    dout = I.make_dout(w.seed + 9000, w.batch, w.L, w.heads, w.head_dim)
    p, got, idx = _gpu_bwd(w, x, dout)
    D, R, Hh = w.head_dim, w.rank, w.heads
    A = oracle.decode_bf16(x["A"]).reshape(D, R)
    grid = (w.T, w.H, w.W)
    h = 5
    rng = np.random.default_rng(13)
    qbs = sorted({0, w.nb - 1, *rng.choice(w.nb, 2, replace=False).tolist()})
    counts = np.bincount(idx[h].ravel(), minlength=w.nb)
    kbs = sorted({0, w.nb - 1, int(counts.argmax())})
    dA_ref = np.zeros((D, R))
    for hh in range(Hh):
        r = OB.head_backward_sampled(oracle.decode_bf16(x["q"][0, :, hh]), oracle.decode_bf16(x["k"][0, :, hh]),
                                     oracle.decode_bf16(x["v"][0, :, hh]), A, dout[0, :, hh].astype(np.float64),
                                     grid, w.block, R, idx[hh], qbs if hh == h else [], kbs if hh == h else [])
        dA_ref += r["dA"]
        if hh == h:
            smp = r
    rows = lambda a: slice(a * w.block, min(w.L, (a + 1) * w.block))
    got_s = [np.concatenate([got[0][0, rows(a), h] for a in qbs]), np.concatenate([got[1][0, rows(b), h] for b in kbs]),
             np.concatenate([got[2][0, rows(b), h] for b in kbs]), got[3]]
    ref_s = [np.concatenate([smp["dq"][a] for a in qbs]), np.concatenate([smp["dk"][b] for b in kbs]),
             np.concatenate([smp["dv"][b] for b in kbs]), dA_ref]
    _compare("wan1.3b-sampled", got_s, ref_s)


def _saved_vs_recompute(w, branches=slra.BRANCH_BOTH):
    """slra_attn_fwd_train gives slra_attn_fwd_ex's output bit for bit, and slra_attn_bwd_saved on its
    workspace gives slra_attn_bwd's gradients bit for bit (the saved O_s and lse are the ones the
    recompute writes: same kernel, same arithmetic)."""
    import torch
    x = I.make_inputs(w)
    dout = torch.from_numpy(I.make_dout(w.seed + 9100, w.batch, w.L, w.heads, w.head_dim)).cuda()
    p = slra.Problem.from_workload(w, branches=branches)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    out_ref, ws_f = slra.attn_fwd(p, q, k, v, A)
    assert slra.device_status(ws_f) == slra.OK
    out_t, ws = slra.attn_fwd_train(p, q, k, v, A)
    assert slra.device_status(ws) == slra.OK
    assert torch.equal(out_t, out_ref)
    ref = slra.attn_bwd(p, q, k, v, A, dout)[:4]
    got = slra.attn_bwd_saved(p, q, k, v, A, dout, ws)[:4]
    assert slra.device_status(ws) == slra.OK
    for name, a, b in zip(("dq", "dk", "dv", "dA"), got, ref):
        assert torch.equal(a, b), f"{w.name}: {name} differs from the recomputing backward"


@pytest.mark.parametrize("w", [W.TINY, EDGE_128, EDGE_128_B64, EDGE_B2, W.WAN_1_3B], ids=lambda w: w.name)
def test_saved_forward_backward_equals_recompute(w):
    _saved_vs_recompute(w)


@pytest.mark.parametrize("branches", [slra.BRANCH_SPARSE, slra.BRANCH_LOWRANK])
def test_saved_forward_backward_single_branch(branches):
    _saved_vs_recompute(EDGE_128, branches)


# ---- the forward's options (RoLA 5.3 Table 6 feature maps, the RoPE orderings of Table 2, separate and
# per-head projections of App. E.2 / RoPeSLR's head-wise parameterization)

R128 = W.Workload("bwd-r128", 1, 2, 128, 2, 9, 11, 128, 64, 0.25, 7500)    # rank 128: untiled fp32 passes
EDGE_PROJ = W.Workload("bwd-proj-128", 1, 8, 128, 4, 24, 32, 32, 128, 0.1, 7300)  # CTAs change head


def _nonneg(x):
    """q, k and A with the bf16 sign bit cleared, so every feature x A >= 0 and the normaliser stays
    away from zero for the maps whose features can be negative (as in the forward's tests)."""
    y = dict(x)
    for n in ("q", "k", "A"):
        y[n] = np.bitwise_and(x[n], np.uint16(0x7FFF))
    return y


def _case_opts(w, label, activation=slra.ACT_RELU, rope="outside", separate=0, per_head=0,
               branches=slra.BRANCH_BOTH, nonneg=False):
    x = I.make_inputs(w)
    if separate or per_head:
        x["A"] = I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, bool(separate), bool(per_head))
    if nonneg:
        x = _nonneg(x)
    dout = I.make_dout(w.seed + 9000, w.batch, w.L, w.heads, w.head_dim)
    kw = dict(branches=branches, activation=activation, lowrank_norope=int(rope == "none"),
              lowrank_rope_inside=int(rope == "inside"), proj_separate=separate, proj_per_head=per_head)
    p, got, idx = _gpu_bwd(w, x, dout, **kw)
    ref = _oracle_bwd(w, x, dout, idx, branches, activation, rope, separate, per_head)
    return _compare(label, got, ref)


@pytest.mark.parametrize("act", [slra.ACT_SILU, slra.ACT_IDENTITY, slra.ACT_TANH])
@pytest.mark.parametrize("w", [W.TINY, EDGE_128, EDGE_128_B64, R128], ids=lambda w: w.name)
def test_backward_activations(w, act):
    """Each feature map on every low-rank gradient path: head_dim 64 and rank 64 (register-tiled fp32),
    rank 32 (tensor cores), rank 128 (untiled fp32)."""
    _case_opts(w, f"{w.name}-act{act}", activation=act, nonneg=True)


@pytest.mark.parametrize("rope", ["none", "inside"])
@pytest.mark.parametrize("w", [W.TINY, EDGE_128, EDGE_128_B64, R128], ids=lambda w: w.name)
def test_backward_rope_orderings(w, rope):
    """No low-rank RoPE, and the RoPE inside the activation (the normaliser on psi), on every path;
    inside with SiLU on the tensor-core path."""
    _case_opts(w, f"{w.name}-rope-{rope}", rope=rope)
    if rope == "inside" and w is EDGE_128:
        _case_opts(w, f"{w.name}-rope-inside-silu", rope=rope, activation=slra.ACT_SILU, nonneg=True)


@pytest.mark.parametrize("separate,per_head", [(1, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("w", [W.TINY, EDGE_128, EDGE_128_B64, R128, EDGE_PROJ], ids=lambda w: w.name)
def test_backward_projections(w, separate, per_head):
    """Separate query / key projections and per-head projections: dA per projection in the argument's
    layout, on every path; 8 heads on the tensor-core path, where persistent CTAs restage the head's
    projection between work items."""
    _case_opts(w, f"{w.name}-proj-s{separate}-h{per_head}", separate=separate, per_head=per_head)


def test_backward_r128_default():
    _case_opts(R128, "bwd-r128")


def test_saved_backward_with_options():
    """The training pair with SiLU features and separate per-head projections: bit for bit the
    recomputing backward."""
    import torch
    w = EDGE_PROJ
    x = _nonneg(dict(I.make_inputs(w), A=I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, True, True)))
    dout = torch.from_numpy(I.make_dout(w.seed + 9100, w.batch, w.L, w.heads, w.head_dim)).cuda()
    p = slra.Problem.from_workload(w, activation=slra.ACT_SILU, proj_separate=1, proj_per_head=1)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    out_ref = slra.attn_fwd(p, q, k, v, A)[0]
    out_t, ws = slra.attn_fwd_train(p, q, k, v, A)
    assert torch.equal(out_t, out_ref)
    ref = slra.attn_bwd(p, q, k, v, A, dout)[:4]
    got = slra.attn_bwd_saved(p, q, k, v, A, dout, ws)[:4]
    assert slra.device_status(ws) == slra.OK
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


# ---- the gated fusion (RoLA 4.4 as the forward reads it): gradients of q, k, v, A and of Wg, bg

def _gate_params(w, bias, seed=77):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(w.head_dim) / np.sqrt(w.head_dim)).astype(np.float32), float(bias)


def _gated_case(w, label, bias, activation=slra.ACT_RELU, separate=0, per_head=0, nonneg=False):
    import torch
    import oracle
    from oracle import backward as OB
    x = I.make_inputs(w)
    if separate or per_head:
        x["A"] = I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, bool(separate), bool(per_head))
    if nonneg:
        x = _nonneg(x)
    gw, gb = _gate_params(w, bias)
    dout = I.make_dout(w.seed + 9000, w.batch, w.L, w.heads, w.head_dim)
    dgw = torch.empty(w.head_dim, dtype=torch.float32, device="cuda")
    dgb = torch.empty(1, dtype=torch.float32, device="cuda")
    p = slra.Problem.from_workload(w, fusion=slra.FUSION_GATED, gate_bias=gb, gate_w=torch.from_numpy(gw).cuda(),
                                   activation=activation, proj_separate=separate, proj_per_head=per_head,
                                   dgate_w=dgw, dgate_b=dgb)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    dq, dk, dv, dA, ws = slra.attn_bwd(p, q, k, v, A, torch.from_numpy(dout).cuda())
    assert slra.device_status(ws) == slra.OK
    idx = slra.ws_view(p, ws, "idx").cpu().numpy()
    got = [t.cpu().numpy().astype(np.float64) for t in (dq, dk, dv, dA)]
    B, L, Hh, D = x["q"].shape
    nh = Hh if per_head else 1
    P = oracle.decode_bf16(x["A"]).reshape(1 + separate, nh, D, w.rank)
    ref = [np.zeros((B, L, Hh, D)) for _ in range(3)] + [np.zeros((1 + separate, nh, D, w.rank))]
    rgw, rgb = np.zeros(D), 0.0
    for b in range(B):
        for h in range(Hh):
            hp = h if per_head else 0
            r = OB.head_backward(oracle.decode_bf16(x["q"][b, :, h]), oracle.decode_bf16(x["k"][b, :, h]),
                                 oracle.decode_bf16(x["v"][b, :, h]), P[0, hp], dout[b, :, h].astype(np.float64),
                                 (w.T, w.H, w.W), w.block, w.keep_frac, w.rank, idx=idx[b * Hh + h],
                                 activation=activation, A_k=P[1, hp] if separate else None,
                                 gate=(gw.astype(np.float64), gb))
            ref[0][b, :, h], ref[1][b, :, h], ref[2][b, :, h] = r["dq"], r["dk"], r["dv"]
            ref[3][0, hp] += r["dA"]
            if separate:
                ref[3][1, hp] += r["dA_k"]
            rgw += r["dgate_w"]
            rgb += float(r["dgate_b"])
    if not separate and not per_head:
        ref[3] = ref[3].reshape(D, w.rank)
    _compare(label, got, ref)
    # [dWg, dbg] as one vector (compared under the first name of the report)
    _compare(label + "-gate", [np.concatenate([dgw.cpu().numpy().astype(np.float64), dgb.cpu().numpy()])],
             [np.concatenate([rgw, [rgb]])])
    return p, (q, k, v, A), dout


@pytest.mark.parametrize("bias", [-2.0, 0.5])
@pytest.mark.parametrize("w", [W.TINY, EDGE_128, EDGE_128_B64], ids=lambda w: w.name)
def test_backward_gated_fusion(w, bias):
    """dq, dk, dv, dA and the gate's dWg, dbg on every low-rank path, a closed-ish and an open gate."""
    _gated_case(w, f"{w.name}-gated{bias}", bias)


def test_backward_gated_with_other_options():
    """The gate together with SiLU features and separate per-head projections (8 heads, tensor cores)."""
    _gated_case(EDGE_PROJ, "proj-gated-silu", -1.0, activation=slra.ACT_SILU, separate=1, per_head=1, nonneg=True)


def test_saved_backward_gated():
    """The training pair with the gated fusion: forward output and every gradient bit for bit those of
    the forward and the recomputing backward."""
    import torch
    w = EDGE_128
    x = I.make_inputs(w)
    gw, gb = _gate_params(w, -1.0)
    dout = torch.from_numpy(I.make_dout(w.seed + 9100, w.batch, w.L, w.heads, w.head_dim)).cuda()
    g1 = (torch.empty(w.head_dim, device="cuda"), torch.empty(1, device="cuda"))
    g2 = (torch.empty(w.head_dim, device="cuda"), torch.empty(1, device="cuda"))
    kw = dict(fusion=slra.FUSION_GATED, gate_bias=gb, gate_w=torch.from_numpy(gw).cuda())
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    p1 = slra.Problem.from_workload(w, dgate_w=g1[0], dgate_b=g1[1], **kw)
    p2 = slra.Problem.from_workload(w, dgate_w=g2[0], dgate_b=g2[1], **kw)
    out_ref = slra.attn_fwd(p1, q, k, v, A)[0]
    out_t, ws = slra.attn_fwd_train(p2, q, k, v, A)
    assert torch.equal(out_t, out_ref)
    ref = slra.attn_bwd(p1, q, k, v, A, dout)[:4]
    got = slra.attn_bwd_saved(p2, q, k, v, A, dout, ws)[:4]
    assert slra.device_status(ws) == slra.OK
    for a, b in zip(got + g2, ref + g1):
        assert torch.equal(a, b)


def test_backward_gated_batch2():
    """The gate's dWg and dbg sum over batch elements and heads: batch 2, three heads."""
    _gated_case(EDGE_B2, "edge-b2-gated", -0.5)


def test_saved_backward_bf16_output():
    """The training forward with a bf16 output: the output bit for bit the forward's, the kept O_s and
    lse (fp32 regardless of the output type) give the recomputing backward's gradients bit for bit."""
    import torch
    w = EDGE_128
    x = I.make_inputs(w)
    dout = torch.from_numpy(I.make_dout(w.seed + 9200, w.batch, w.L, w.heads, w.head_dim)).cuda()
    p = slra.Problem.from_workload(w, out_dtype=slra.OUT_BF16)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    out_ref = slra.attn_fwd(p, q, k, v, A)[0]
    out_t, ws = slra.attn_fwd_train(p, q, k, v, A)
    assert out_t.dtype == torch.bfloat16 and torch.equal(out_t, out_ref)
    ref = slra.attn_bwd(p, q, k, v, A, dout)[:4]
    got = slra.attn_bwd_saved(p, q, k, v, A, dout, ws)[:4]
    assert slra.device_status(ws) == slra.OK
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
