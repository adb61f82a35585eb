"""GPU parity: the C-ABI CUDA path against the fp64 oracle on the same seeded inputs.

Small cases are compared element by element over every output; the large workloads (the
configurations the benchmark times) on every mask row and S/z of sampled heads and on the outputs of
sampled query blocks (first, last = ragged, and random ones).  Tolerances are in tests/parity.py.
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

# Optional per-case error statistics (JSON lines), written when SLRA_PARITY_REPORT names a file.
REPORT = os.environ.get("SLRA_PARITY_REPORT")


def _log(stats):
    if not REPORT:
        return
    try:
        if os.path.dirname(REPORT):
            os.makedirs(os.path.dirname(REPORT), exist_ok=True)
        with open(REPORT, "a") as f:
            f.write(json.dumps({k: (float(v) if isinstance(v, (np.floating,)) else v) for k, v in stats.items()}) + "\n")
    except OSError:
        pass


@pytest.fixture(scope="module", autouse=True)
def _build():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_rank_hybrid_b200 import build
    build.build()
    import oracle
    oracle.build()


def _case(w, label=None, heads=None, qblocks=None, transform=None, **kw):
    p = slra.Problem.from_workload(w, **kw)
    x = I.make_inputs(w)
    if transform is not None:
        x = transform(x)
    gpu = parity.run_gpu(p, x)
    st = parity.compare(p, x, gpu, heads=heads, qblocks=qblocks, label=label or w.name)
    _log(st)
    return st, gpu


def test_tiny_full():
    _case(W.TINY)


def test_tiny_branches_separately():
    _case(W.TINY, "tiny-sparse-only", branches=slra.BRANCH_SPARSE)
    _case(W.TINY, "tiny-lowrank-only", branches=slra.BRANCH_LOWRANK)


@pytest.mark.parametrize("grid,D,R,block,keep,B,heads", [
    ((3, 10, 13), 128, 32, 128, 0.3, 1, 2),    # L = 390: ragged last block (6 tokens)
    ((2, 9, 11), 64, 64, 64, 0.25, 2, 3),      # batch 2, D = 64, r = D, ragged (6 tokens)
    ((1, 5, 7), 128, 16, 128, 0.1, 1, 1),      # L < block: one block, k = 1
    ((4, 12, 16), 128, 128, 128, 1.0, 1, 2),   # keep everything: dense attention, r = D
    ((4, 12, 16), 128, 64, 64, 0.05, 1, 2),    # block 64 with D = 128, keep = 1 of 12
    ((5, 16, 20), 128, 48, 128, 0.2, 1, 3),    # r = 48 (not a power of two)
])
def test_edge_shapes(grid, D, R, block, keep, B, heads):
    w = W.Workload(f"edge-{grid}-{D}-{R}-{block}-{keep}", B, heads, D, *grid, R, block, keep, 7000 + D + R)
    _case(w)


def _nonneg(x):
    """q, k and A with the bf16 sign bit cleared: every feature x A is then >= 0, which keeps the
    normaliser phi(q) . z + 1e-6 away from zero for the identity and tanh maps."""
    y = dict(x)
    for n in ("q", "k", "A"):
        y[n] = np.bitwise_and(x[n], np.uint16(0x7FFF))
    return y


EDGE_128 = W.Workload("edge-act-128", 1, 2, 128, 3, 10, 13, 32, 128, 0.3, 7160)   # L = 390, ragged
EDGE_128_R64 = W.Workload("edge-act-128-r64", 1, 2, 128, 2, 9, 11, 64, 64, 0.25, 7192)


@pytest.mark.parametrize("act", [slra.ACT_SILU, slra.ACT_IDENTITY, slra.ACT_TANH])
def test_activation_variants(act):
    """The feature map's alternatives (RoLA 5.3, Table 6) on both readout paths: head_dim 64 (CUDA
    cores) and head_dim 128 (tensor cores; r = 32, and r = 64 with block 64).  Features that can be
    negative let the normaliser come close to zero on Gaussian inputs (SiLU on the tiny case: 0.13
    against a median of 159, low-rank outputs up to ~590, where fp32 rounding alone exceeds the 1e-2
    absolute bound), so these cases use non-negative q, k and A."""
    _case(W.TINY, f"tiny-act{act}", activation=act, transform=_nonneg)
    _case(EDGE_128, f"edge128-act{act}", activation=act, transform=_nonneg)
    _case(EDGE_128_R64, f"edge128r64-act{act}", activation=act, transform=_nonneg)


def test_lowrank_without_rope():
    """The low-rank branch without its RoPE (psi = phi) on both readout paths, and with SiLU on a
    sampled head of the Wan2.1-1.3B shape."""
    _case(W.TINY, "tiny-norope", lowrank_norope=1)
    _case(EDGE_128, "edge128-norope", lowrank_norope=1)
    w = W.WAN_1_3B
    _case(w, "wan1.3b-silu-norope", heads=[(0, 5)], qblocks=_sample_blocks(w.nb, 4, n=2),
          activation=slra.ACT_SILU, lowrank_norope=1, transform=_nonneg)


def _identity_A(x):
    """A = I (bf16 1.0 on the diagonal) for a rank equal to head_dim."""
    y = dict(x)
    D = x["A"].shape[0]
    a = np.zeros((D, D), dtype=np.uint16)
    a[np.arange(D), np.arange(D)] = 0x3F80
    y["A"] = a
    return y


def test_full_width_linear_baseline():
    """r = D, A = I, relu, no low-rank RoPE: ReLU linear attention with a D x D context (the
    pages' full-width linear branch), on both readout paths."""
    _case(W.TINY.with_(rank=64), "tiny-linear", lowrank_norope=1, transform=_identity_A)
    _case(EDGE_128.with_(rank=128), "edge128-linear", lowrank_norope=1, transform=_identity_A)


def _projections(w, separate, per_head):
    """Replace A by separate (Pq, Pk) and/or per-head projections drawn for this workload."""
    def t(x):
        y = dict(x)
        y["A"] = I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, bool(separate), bool(per_head))
        return y
    return t


# 8 heads x 24 tiles of 128 tokens = 192 low-rank work items for 148 persistent CTAs, so CTAs take
# items of two different heads and restage the key projection in between
EDGE_PROJ = W.Workload("edge-proj-128", 1, 8, 128, 4, 24, 32, 32, 128, 0.1, 7300)


@pytest.mark.parametrize("separate,per_head", [(1, 0), (0, 1), (1, 1)])
def test_projection_variants(separate, per_head):
    """Separate query / key projections (RoLA E.2's Pq, Pk) and per-head projections (RoPeSLR's
    head-wise parameterization) on both readout paths, including persistent low-rank CTAs that
    change head (and so projection) between work items."""
    for w in (W.TINY, EDGE_128, EDGE_128_R64, EDGE_PROJ):
        _case(w, f"{w.name}-proj-s{separate}-h{per_head}", proj_separate=separate, proj_per_head=per_head,
              transform=_projections(w, separate, per_head))


def test_projection_per_head_wan_1_3b():
    """Separate per-head projections at the Wan2.1-1.3B shape (1536 low-rank work items over 148
    CTAs), on sampled heads and query blocks."""
    w = W.WAN_1_3B
    _case(w, "wan1.3b-proj-s1-h1", heads=[(0, 3), (0, 10)], qblocks=_sample_blocks(w.nb, 9, n=2),
          proj_separate=1, proj_per_head=1, transform=_projections(w, 1, 1))


def _gate(w, bias, seed=77):
    """Gated-fusion options: Wg ~ N(0, 1/D) in fp32 (seeded), the given bias."""
    import torch
    rng = np.random.default_rng(seed)
    gw = (rng.standard_normal(w.head_dim) / np.sqrt(w.head_dim)).astype(np.float32)
    return dict(fusion=slra.FUSION_GATED, gate_bias=bias, gate_w=torch.from_numpy(gw).cuda())


@pytest.mark.parametrize("bias", [-2.0, 0.5, -30.0])
def test_gated_fusion(bias):
    """The gated fusion of the branches (RoLA 4.4 as read here) on both readout paths: a typical
    negative bias, an open gate, and a closed one (the output is then the sparse branch's)."""
    for w in (W.TINY, EDGE_128, EDGE_128_R64):
        _case(w, f"{w.name}-gated{bias}", **_gate(w, bias))


def test_gated_fusion_with_other_options():
    """Gated fusion together with separate per-head projections and SiLU features, and at the
    Wan2.1-1.3B shape on sampled heads and query blocks."""
    _case(EDGE_PROJ, "edge-proj-gated-silu", proj_separate=1, proj_per_head=1, activation=slra.ACT_SILU,
          transform=lambda x: _nonneg(_projections(EDGE_PROJ, 1, 1)(x)), **_gate(EDGE_PROJ, -1.0))
    w = W.WAN_1_3B
    _case(w, "wan1.3b-gated", heads=[(0, 2)], qblocks=_sample_blocks(w.nb, 13, n=2), **_gate(w, -2.0))


def test_rope_inside_activation():
    """The truncated RoPE before the activation (the ordering RoLA's ablation compares against), on
    both readout paths, with persistent summary CTAs changing head, and with SiLU."""
    for w in (W.TINY, EDGE_128, EDGE_128_R64, EDGE_PROJ):
        _case(w, f"{w.name}-inside", lowrank_rope_inside=1)
    _case(EDGE_128, "edge128-inside-silu", lowrank_rope_inside=1, activation=slra.ACT_SILU, transform=_nonneg)


def test_shift_residual_by_rope_ordering():
    """RoLA Table 2's shift residual on synthetic inputs, measured on the GPU path's low-rank branch:
    ||O_lr(p + c) - O_lr(p)|| / ||O_lr(p)|| for a constant shift c.  RoPE outside the activation:
    unchanged up to fp32 rounding of the shifted angles; without RoPE: bit-identical; inside the
    activation: a change of order one (absolute position leaks through the nonlinearity)."""
    w = EDGE_128
    x = I.make_inputs(w)
    res = {}
    for name, kw in (("outside", {}), ("none", {"lowrank_norope": 1}), ("inside", {"lowrank_rope_inside": 1})):
        a = parity.run_gpu(slra.Problem.from_workload(w, branches=slra.BRANCH_LOWRANK, **kw), x)["out"]
        b = parity.run_gpu(slra.Problem.from_workload(w, branches=slra.BRANCH_LOWRANK, pos_offset=(2, 3, 5), **kw),
                           x)["out"]
        res[name] = float(np.linalg.norm(a - b) / np.linalg.norm(a))
    _log({"label": "shift-residual-edge128", **res})
    assert res["outside"] < 1e-4 and res["none"] == 0.0 and res["inside"] > 1e-2


def test_exact_ties_keep_the_lower_blocks():
    """Key blocks whose keys are all zero have block means of exactly zero, so their scores tie exactly
    (+0 for every query block, whose mean has components of both signs); the selection keeps the
    lowest-indexed of the tied blocks, the oracle's rule.  Here the cut falls inside the tied group,
    so every row is tie-flagged and the kept lists must equal the oracle's bit for bit anyway."""
    w = W.TINY.with_(name="ties", T=4, H=16, W=16, heads=2, block=64, keep_frac=0.5)  # 16 blocks, keep 8
    x = I.make_inputs(w)
    k = x["k"].copy()
    k[:, 2 * 64:14 * 64] = 0  # blocks 2..13: zero keys
    x = dict(x, k=k)
    p = slra.Problem.from_workload(w)
    gpu = parity.run_gpu(p, x)
    import oracle
    _, per = oracle.forward(x, (w.T, w.H, w.W), w.block, w.keep_frac, w.rank, branches=1, qblocks=[0])
    for (b, h), r in per.items():
        bh = b * w.heads + h
        assert r["tie"].any()
        assert np.array_equal(gpu["idx"][bh], r["idx"]), (bh, gpu["idx"][bh], r["idx"])
        assert np.array_equal(gpu["tie"][bh].astype(bool), r["tie"].astype(bool))
    parity.compare(p, x, gpu, label="exact-ties")


def test_shift_invariance_on_gpu():
    """Shifting all positions leaves the masks unchanged exactly (fp64 selection) and the outputs
    unchanged up to the fp16 rounding of the rotated operands, which differs between the two runs (the
    same exact values rotated by other angles round differently): measured on a B200, max-abs 1.6e-3 and
    mean-relative 2.4e-4 between the two runs, so the bound between them is 4e-3 / 6e-4; both also stay
    within the parity tolerance of the (exactly invariant) oracle."""
    w = W.TINY.with_(T=4, H=16, W=16, heads=2, block=64, keep_frac=0.25)
    x = I.make_inputs(w)
    p0 = slra.Problem.from_workload(w)
    p1 = slra.Problem.from_workload(w, pos_offset=(3, -7, 11))
    g0, g1 = parity.run_gpu(p0, x), parity.run_gpu(p1, x)
    assert np.array_equal(g0["idx"], g1["idx"])
    d = np.abs(g0["out"] - g1["out"])
    _log({"label": "shift-gpu-vs-gpu", "max_abs": float(d.max()), "mean_rel": float(d.sum() / np.abs(g0["out"]).sum())})
    assert d.max() <= 4e-3 and d.sum() / np.abs(g0["out"]).sum() <= 6e-4
    parity.compare(p1, x, g1, label="tiny-shifted")


def test_deterministic_and_bf16_out():
    w = W.TINY.with_(T=4, H=16, W=16, heads=2, block=64, keep_frac=0.25)
    x = I.make_inputs(w)
    p = slra.Problem.from_workload(w)
    a, b = parity.run_gpu(p, x), parity.run_gpu(p, x)
    assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["idx"], b["idx"])
    pb = slra.Problem.from_workload(w, out_dtype=slra.OUT_BF16)
    c = parity.run_gpu(pb, x)
    # bf16 rounding of the output: at most half an ulp of bf16 (2^-9 relative) plus the fp32 error
    assert np.all(np.abs(c["out"] - a["out"]) <= np.abs(a["out"]) * 2.0 ** -8 + 1e-6)


def test_host_entry_point_matches_device():
    import torch
    w = W.TINY
    x = I.make_inputs(w)
    p = slra.Problem.from_workload(w)
    dev = parity.run_gpu(p, x)["out"]
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v", "A")}
    out = torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32).pin_memory()
    io = torch.empty(slra.host_io_bytes(p), dtype=torch.uint8, device="cuda")
    ws = slra.alloc_workspace(p)
    slra.attn_fwd_host(p, host["q"], host["k"], host["v"], host["A"], out, io, ws)
    assert np.array_equal(out.numpy().astype(np.float64), dev)


def _host_out(p, x):
    import torch
    host = {n: torch.from_numpy(np.ascontiguousarray(x[n]).view(np.int16)).view(torch.bfloat16).pin_memory()
            for n in ("q", "k", "v", "A")}
    dt = torch.float32 if p.out_dtype == slra.OUT_F32 else torch.bfloat16
    out = torch.empty((p.batch, p.L, p.heads, p.head_dim), dtype=dt).pin_memory()
    io = torch.empty(slra.host_io_bytes(p), dtype=torch.uint8, device="cuda")
    ws = slra.alloc_workspace(p)
    assert slra.host_pipeline_groups(p, io.numel(), ws.numel()) > 1  # the pipelined path is the one tested
    slra.attn_fwd_host(p, host["q"], host["k"], host["v"], host["A"], out, io, ws)
    st = slra.device_status(ws)
    assert st == slra.OK, slra.status_string(st)
    return out.float().numpy().astype(np.float64)


EDGE_B2 = W.Workload("edge-b2-128", 2, 5, 128, 2, 9, 11, 32, 64, 0.25, 7410)


@pytest.mark.parametrize("case", ["plain", "options", "batch2", "bf16"])
def test_host_entry_point_pipelined(case):
    """The host entry point's pipelined head groups (uploads, compute and downloads overlapped) give
    the device entry point's output: the same kernels per head, only the low-rank summary's split of
    the sequence can differ with the group size (fp32 order), hence a relative bound instead of
    equality; and the result is within the oracle tolerance."""
    w, kw, tf = EDGE_PROJ, {}, None
    if case == "options":
        kw = dict(proj_separate=1, proj_per_head=1, activation=slra.ACT_SILU, **_gate(EDGE_PROJ, -1.0))
        tf = lambda x: _nonneg(_projections(EDGE_PROJ, 1, 1)(x))
    elif case == "batch2":
        w = EDGE_B2
    elif case == "bf16":
        kw = dict(out_dtype=slra.OUT_BF16)
    p = slra.Problem.from_workload(w, **kw)
    x = I.make_inputs(w)
    if tf is not None:
        x = tf(x)
    dev = parity.run_gpu(p, x)
    host = _host_out(p, x)
    assert np.abs(host - dev["out"]).max() <= 1e-5 * np.abs(dev["out"]).max() + (4e-3 if case == "bf16" else 0.0)
    if case != "bf16":
        dev["out"] = host
        _log(parity.compare(p, x, dev, label=f"host-pipelined-{case}"))


def _rescaled(x, seed, q=1.0, k=1.0, v=1.0, q_uniform=None):
    """Inputs with q, k, v multiplied by the given factors and re-rounded to bf16 (RNE); q_uniform = c
    draws q uniform in [-c, c] instead (seeded), so |q| stays below c and a rotated pair below c*sqrt(2)."""
    y = dict(x)
    for n, f in (("q", q), ("k", k), ("v", v)):
        if f != 1.0:
            y[n] = I.f32_to_bf16_bits(I.bf16_bits_to_f32(x[n]) * np.float32(f))
    if q_uniform is not None:
        rng = np.random.default_rng(seed)
        y["q"] = I.f32_to_bf16_bits(rng.uniform(-q_uniform, q_uniform, x["q"].shape).astype(np.float32))
    return y


# (label, factors, absolute-bound multiplier): inputs far from unit scale, where the fp16 operands of
# the attention kernel could lose range or precision.  q near 45,000 with k near 1e-4 keeps the logits
# of order one while the rotated queries come within 3% of fp16's largest finite value (65,504).
SCALE_CASES = [
    ("qkv-1e-3", dict(q=1e-3, k=1e-3, v=1e-3), 1.0),
    ("qkv-1e-5", dict(q=1e-5, k=1e-5, v=1e-5), 1.0),  # below fp16's normal range: reported (see below)
    ("v-1e-4", dict(v=1e-4), 1.0),
    ("v-300", dict(v=300.0), 300.0),
    ("q-near-fp16-max", dict(k=1e-4, q_uniform=45000.0), 1.0),
]


@pytest.mark.parametrize("label,factors,abs_mult", SCALE_CASES, ids=[c[0] for c in SCALE_CASES])
@pytest.mark.parametrize("D", [64, 128])
def test_input_scales(label, factors, abs_mult, D):
    """Element-by-element parity far from unit scale (RoLA 4.1 defines the method on the model's
    activations, which are not normalised), on both head dims; the device status must stay clean."""
    w = W.Workload(f"scale-{label}-{D}", 1, 2, D, 3, 10, 13, 32 if D == 128 else 16, 64, 0.3, 7500 + D)
    x = _rescaled(I.make_custom(w.seed, 1, (w.T, w.H, w.W), w.heads, D, w.rank), w.seed + 1, **factors)
    p = slra.Problem.from_workload(w)
    # blocks whose values all sit below fp16's smallest normal (2^-14) are reported as a range problem
    # (the fp16 copies keep only absolute precision there); the result is still compared
    expect = slra.ERR_RANGE if label == "qkv-1e-5" else slra.OK
    gpu = parity.run_gpu(p, x, expect_status=expect)
    _log(parity.compare(p, x, gpu, label=f"scale-{label}-{D}", max_abs=parity.MAX_ABS * abs_mult))


def test_range_error_reported():
    """An input too large for the fp16 operands is reported through the device status word."""
    import torch
    w = W.TINY
    x = I.make_inputs(w)
    q = parity.to_gpu(x["q"]).clone()
    q[0, 5, 0, 3] = 1e6
    k, v, A = (parity.to_gpu(x[n]) for n in ("k", "v", "A"))
    p = slra.Problem.from_workload(w)
    _, ws = slra.attn_fwd(p, q, k, v, A)
    assert slra.device_status(ws) == slra.ERR_RANGE
    assert slra.device_status(ws) == slra.OK  # reading clears it


def _sample_blocks(nb, seed, n=3):
    rng = np.random.default_rng(seed)
    return sorted({0, nb - 1, *rng.choice(nb, size=n, replace=False).tolist()})


def test_wan_1_3b_full_size():
    w = W.WAN_1_3B
    heads = [(0, 0), (0, 5), (0, 11)]
    _case(w, heads=heads, qblocks=_sample_blocks(w.nb, 1))


def test_wan_14b_bench_config():
    """The configuration the benchmark times (Wan2.1-14B 720p, 75,600 tokens, 40 heads, keep 10%)."""
    w = W.WAN_14B
    heads = [(0, 0), (0, 17), (0, 39)]
    _case(w, heads=heads, qblocks=_sample_blocks(w.nb, 2))


@pytest.mark.slow
def test_hunyuan_long():
    w = W.HUNYUAN
    heads = [(0, 0), (0, 23)]
    _case(w, heads=heads, qblocks=_sample_blocks(w.nb, 3, n=2))


@pytest.mark.parametrize("name", ["sweep-keep5-r16", "sweep-keep100-r128", "sweep-keep50-r64"])
def test_sweep_points(name):
    w = W.by_name(name)
    heads = [(0, 3)]
    _case(w, heads=heads, qblocks=[0, w.nb - 1])


def test_bounded_wait_timeout_is_reported_and_context_stays_usable():
    """A wait on a barrier that nothing signals runs out after its bound, the kernel records a timeout
    in the status word and returns without issuing work; the next call on the same context is exact."""
    w = W.TINY
    x = I.make_inputs(w)
    q, k, v, A = (parity.to_gpu(x[n]) for n in ("q", "k", "v", "A"))
    p = slra.Problem.from_workload(w, debug_flags=slra.DEBUG_UNSATISFIED_WAIT, wait_timeout_ns=1_000_000)
    _, ws = slra.attn_fwd(p, q, k, v, A)
    assert slra.device_status(ws) == slra.ERR_DEVICE_TIMEOUT
    assert slra.device_status(ws) == slra.OK
    st = parity.compare(slra.Problem.from_workload(w), x, parity.run_gpu(slra.Problem.from_workload(w), x),
                        label="tiny-after-timeout")
    _log(st)
