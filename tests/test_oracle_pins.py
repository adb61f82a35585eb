"""Pins of the fp64 oracle against facts fixed by the definitions and the mathematics (CPU only).

Each test names what it pins and which plausible mistake it would catch.  Sources: RoLA
("3 Preliminary" 3D RoPE and eq. (1) relative property; "4.1" block-sparse + low-rank branches;
"4.2" rank-truncated rotary schedule; "4.3"/"B.1" RoPE outside the activation, one query-independent
sum; "B.2" geometric rotary schedule) and RoPeSLR's appendix on 3D RoPE (base 10000).
"""
import math
import os

import numpy as np
import pytest

from tests import brute
from sparse_rank_hybrid_b200 import inputs as I
from sparse_rank_hybrid_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(path):
    with open(path) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


# ------------------------------------------------------------------------------------ bf16 inputs
def _bf16_golden():
    """(bits, value) pairs of tests/golden/bf16_decode.txt (written by hand from the bf16 format)."""
    bits, vals = [], []
    for h, v in _rows(os.path.join(GOLD, "bf16_decode.txt")):
        bits.append(int(h, 16))
        vals.append(-0.0 if v == "neg0" else float(v))
    return np.array(bits, dtype=np.uint16), np.array(vals, dtype=np.float64)


def _same_values(a, b):
    """Equal as IEEE values, including the sign of zero and NaN in the same places."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    nan = np.isnan(a)
    return bool(np.array_equal(nan, np.isnan(b)) and np.array_equal(a[~nan], b[~nan]) and
                np.array_equal(np.signbit(a[~nan]), np.signbit(b[~nan])))


def _bf16_by_fields(bits):
    """The bf16 definition written out: sign, 8-bit exponent (bias 127), 7-bit fraction, subnormals,
    infinities and NaN (independent of any reinterpretation of memory)."""
    out = []
    for b in np.asarray(bits, dtype=np.uint16).ravel().tolist():
        s, e, f = b >> 15, (b >> 7) & 0xFF, b & 0x7F
        if e == 0xFF:
            x = math.nan if f else math.inf
        elif e == 0:
            x = math.ldexp(f / 128.0, -126)
        else:
            x = math.ldexp(1.0 + f / 128.0, e - 127)
        out.append(-x if s else x)
    return np.array(out, dtype=np.float64).reshape(np.shape(bits))


def test_decode_bf16_golden_table(oracle_mod):
    """orc_decode_bf16 (the entry of every bf16 input into the oracle) returns the exact value of each
    pattern of a hand-written table: signed zeros, +-1, powers of two, the largest finite value, the
    smallest normal, subnormals, infinities and NaN."""
    bits, vals = _bf16_golden()
    assert _same_values(oracle_mod.decode_bf16(bits), vals)
    assert _same_values(_bf16_by_fields(bits), vals)


def test_decode_bf16_all_patterns_and_generator_bits(oracle_mod):
    """All 65,536 patterns against the field-by-field definition and against torch's own bf16 -> fp64
    conversion; then the seeded generator's actual q, k, v and A bits against numpy's reinterpretation
    of the pattern as the upper half of an fp32."""
    torch = pytest.importorskip("torch")
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle_mod.decode_bf16(allb)
    assert _same_values(got, _bf16_by_fields(allb))
    assert _same_values(got, torch.from_numpy(allb.view(np.int16)).view(torch.bfloat16).double().numpy())
    x = I.make_inputs(W.TINY)
    for n in ("q", "k", "v", "A"):
        ref = (x[n].astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        assert _same_values(oracle_mod.decode_bf16(x[n]), ref), n


def test_decode_bf16_pins_reject_planted_mistakes(oracle_mod):
    """Plausible decoder mistakes, planted in CPU decoders written here, fail the golden table:
    shifting by 15 instead of 16, dropping the sign bit, and reading the pattern as fp16."""
    bits, vals = _bf16_golden()
    shift15 = (bits.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)
    unsigned = oracle_mod.decode_bf16(bits & np.uint16(0x7FFF))
    as_fp16 = bits.view(np.float16).astype(np.float64)
    for bad in (shift15, unsigned, as_fp16):
        assert not _same_values(bad, vals)


# ----------------------------------------------------------------------------------------- RoPE
def test_rope_split_golden(oracle_mod):
    """Pairs per axis match the Wan 44/42/42 split (D=128) and the same rule at D=64."""
    for D, pt, ph, pw in _rows(os.path.join(GOLD, "rope_split.txt")):
        axis, _ = oracle_mod.rope_pairs(int(D))
        assert [int((axis == a).sum()) for a in range(3)] == [int(pt), int(ph), int(pw)]
        # native order: all t pairs, then h, then w
        assert np.all(np.diff(axis) >= 0)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_frequencies_geometric_base(oracle_mod, D):
    """Per axis: first frequency 1, constant ratio (geometric, RoLA B.2), and p_a steps of the ratio
    divide by exactly the base 10000 (RoFormer schedule theta^(-2m/d_a)).  Catches a wrong exponent
    width (D instead of d_a), an off-by-one in m, or a wrong base."""
    axis, omega = oracle_mod.rope_pairs(D, theta=1e4)
    for a in range(3):
        w = omega[axis == a]
        p = w.size
        assert w[0] == 1.0
        ratio = w[1:] / w[:-1]
        assert np.allclose(ratio, ratio[0], rtol=1e-13)
        assert math.isclose(ratio[0] ** p, 1e-4, rel_tol=1e-12)


def test_rope_axis_isolation(oracle_mod):
    """With a grid that is 1 long on an axis, that axis' pairs are untouched; with the other two axes
    flat, only that axis' pairs move.  Catches a wrong pair->axis assignment or a wrong token->(t,h,w)
    decomposition."""
    rng = np.random.default_rng(0)
    D = 128
    axis, _ = oracle_mod.rope_pairs(D)
    for a, grid in enumerate([(1, 5, 7), (5, 1, 7), (5, 7, 1)]):
        L = grid[0] * grid[1] * grid[2]
        x = rng.standard_normal((L, D))
        y = oracle_mod.rope_rows(x, grid, D // 2)
        pairs = np.where(axis == a)[0]
        cols = np.sort(np.concatenate([2 * pairs, 2 * pairs + 1]))
        assert np.array_equal(y[:, cols], x[:, cols])
    for a, grid in enumerate([(9, 1, 1), (1, 9, 1), (1, 1, 9)]):
        x = rng.standard_normal((9, D))
        y = oracle_mod.rope_rows(x, grid, D // 2)
        moved = np.where(np.any(y != x, axis=0))[0] // 2
        assert set(np.unique(moved)) <= set(np.where(axis == a)[0])


def test_rope_position_closed_form(oracle_mod):
    """A unit vector in the first pair of an axis (frequency 1) at token (t, h, w) ends at angle
    t (resp. h, w): cos/sin of the integer position, counter-clockwise.  Catches a sign flip of sin,
    a swapped pair layout, or a wrong row-major decomposition."""
    D = 64
    grid = (3, 4, 5)
    axis, _ = oracle_mod.rope_pairs(D)
    first = [int(np.where(axis == a)[0][0]) for a in range(3)]
    L = 60
    x = np.zeros((L, D))
    for j in first:
        x[:, 2 * j] = 1.0
    y = oracle_mod.rope_rows(x, grid, D // 2)
    for n in range(L):
        t, h, w = n // 20, (n // 5) % 4, n % 5
        for a, p in zip(range(3), (t, h, w)):
            j = first[a]
            assert math.isclose(y[n, 2 * j], math.cos(p), abs_tol=1e-15)
            assert math.isclose(y[n, 2 * j + 1], math.sin(p), abs_tol=1e-15)


def test_rope_matches_complex_rotation(oracle_mod):
    """2x2 rotation == complex multiplication by exp(i angle) (independent formulation), including a
    position offset and a truncated rotation (npairs < D/2)."""
    rng = np.random.default_rng(1)
    D, grid, off = 128, (3, 6, 7), (2, -3, 5)
    L = 126
    x = rng.standard_normal((L, D))
    axis, omega = oracle_mod.rope_pairs(D)
    pos = brute.grid_positions(grid, off)
    for npairs in (D // 2, 16, 32):
        y = oracle_mod.rope_rows(x, grid, npairs, offset=off)
        yb = brute.rope_complex(x, pos, axis, omega, npairs)
        assert np.allclose(y, yb, rtol=0, atol=1e-13)


def test_rope_orthogonal_and_relative(oracle_mod):
    """Rotations preserve norms, and q^(p) . k^(p') depends only on p - p' (RoLA eq. (1))."""
    rng = np.random.default_rng(2)
    D, grid = 128, (4, 5, 6)
    L = 120
    q = rng.standard_normal((L, D))
    k = rng.standard_normal((L, D))
    qh = oracle_mod.rope_rows(q, grid, D // 2)
    assert np.allclose(np.linalg.norm(qh, axis=1), np.linalg.norm(q, axis=1), rtol=1e-13)
    s0 = oracle_mod.rope_rows(q, grid, D // 2) @ oracle_mod.rope_rows(k, grid, D // 2).T
    s1 = oracle_mod.rope_rows(q, grid, D // 2, offset=(7, -2, 11)) @ \
        oracle_mod.rope_rows(k, grid, D // 2, offset=(7, -2, 11)).T
    assert np.allclose(s0, s1, rtol=0, atol=1e-10)


# ------------------------------------------------------------------------------ pooling, top-k
def test_block_means_ragged(oracle_mod):
    """Block means == numpy reshape-mean, with a partial last block averaged over its real tokens."""
    rng = np.random.default_rng(3)
    L, D, b = 300, 16, 64
    x = rng.standard_normal((L, D))
    m = oracle_mod.block_means(x, b)
    assert m.shape == (5, D)
    ref = [x[i * b:min(L, (i + 1) * b)].mean(axis=0) for i in range(5)]
    assert np.allclose(m, np.stack(ref), rtol=0, atol=1e-14)
    s = oracle_mod.block_scores(m, m[::-1].copy())
    assert np.allclose(s, m @ m[::-1].T, rtol=0, atol=1e-13)


def test_keep_count_golden(oracle_mod):
    for nb, kf, k in _rows(os.path.join(GOLD, "keep_counts.txt")):
        assert oracle_mod.keep_count(float(kf), int(nb)) == int(k)


@pytest.mark.parametrize("nb,k", [(37, 4), (64, 1), (20, 20), (100, 13)])
def test_topk_matches_full_sort(oracle_mod, nb, k):
    """Top-k by comparator sort == full lexicographic sort, with many exact ties (quantised scores)
    so the lower-index tie-break is exercised; tie flags follow their definition."""
    rng = np.random.default_rng(nb * 7 + k)
    s = np.round(rng.standard_normal((nb, nb)) * 3) / 3  # heavy exact ties
    idx, tie = oracle_mod.topk(s, k)
    assert np.array_equal(idx, brute.topk_lexsort(s, k))
    for a in range(nb):
        srt = np.sort(s[a])[::-1]
        exp = k < nb and (srt[k - 1] - srt[k]) <= 1e-6 * max(1.0, abs(srt[k - 1]))
        assert bool(tie[a]) == bool(exp)


def test_topk_tie_break_prefers_lower_index(oracle_mod):
    s = np.zeros((6, 6))
    s[0] = [1.0, 5.0, 5.0, 2.0, 5.0, 0.5]
    idx, tie = oracle_mod.topk(s, 2)
    assert idx[0].tolist() == [1, 2] and tie[0] == 1
    idx, tie = oracle_mod.topk(s, 3)
    assert idx[0].tolist() == [1, 2, 4] and tie[0] == 0


# --------------------------------------------------------------------------------- sparse branch
def _head(oracle_mod, w, b=0, h=0, **kw):
    x = I.make_inputs(w)
    dec = oracle_mod.decode_bf16
    return oracle_mod.head_forward(dec(x["q"][b, :, h]), dec(x["k"][b, :, h]), dec(x["v"][b, :, h]),
                                   dec(x["A"]), (w.T, w.H, w.W), w.block, w.keep_frac, w.rank, **kw), x


def test_sparse_keep_all_equals_dense_sdpa(oracle_mod):
    """keep_frac = 1: the sparse branch is dense softmax attention (torch fp64 SDPA)."""
    w = W.TINY.with_(keep_frac=1.0)
    r, x = _head(oracle_mod, w, branches=1)
    v = oracle_mod.decode_bf16(x["v"][0, :, 0])
    allowed = np.ones((w.L, w.L), dtype=bool)
    ref = brute.masked_dense_attention(r["qh"], r["kh"], v, allowed)
    assert r["keep"] == 4
    assert np.allclose(r["out_sparse"], ref, rtol=0, atol=1e-12)


def test_sparse_equals_masked_dense_ragged(oracle_mod):
    """keep < 1 on a grid whose L is not a multiple of the block (ragged last block): the gathered-key
    attention equals a dense masked SDPA built from the kept-block mask."""
    grid = (3, 5, 7)  # L = 105, block 32 -> 4 blocks, last has 9 tokens
    x = I.make_custom(11, 1, grid, 1, 64, 16)
    dec = oracle_mod.decode_bf16
    q, k, v, A = dec(x["q"][0, :, 0]), dec(x["k"][0, :, 0]), dec(x["v"][0, :, 0]), dec(x["A"])
    r = oracle_mod.head_forward(q, k, v, A, grid, 32, 0.5, 16, branches=1)
    allowed = brute.block_mask(r["idx"], 105, 32)
    ref = brute.masked_dense_attention(r["qh"], r["kh"], v, allowed)
    assert np.allclose(r["out_sparse"], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------- low-rank branch
def test_features_relu_matmul(oracle_mod):
    import torch
    rng = np.random.default_rng(4)
    x, A = rng.standard_normal((50, 64)), rng.standard_normal((64, 16))
    ref = torch.relu(torch.from_numpy(x) @ torch.from_numpy(A)).numpy()
    assert np.allclose(oracle_mod.features(x, A), ref, rtol=0, atol=1e-13)


def test_features_activation_variants(oracle_mod):
    """The ablation's activations (RoLA 5.3, Table 6) against torch's own SiLU / tanh and a plain
    matmul for identity, plus two closed-form facts of SiLU (catches a sigmoid in place of SiLU, a
    sign flip in the exponent, or an activation applied before the projection)."""
    import torch
    rng = np.random.default_rng(14)
    x, A = rng.standard_normal((40, 64)), rng.standard_normal((64, 16))
    u = torch.from_numpy(x) @ torch.from_numpy(A)
    assert np.allclose(oracle_mod.features(x, A, oracle_mod.ACT_SILU), torch.nn.functional.silu(u).numpy(),
                       rtol=1e-14, atol=1e-14)
    assert np.allclose(oracle_mod.features(x, A, oracle_mod.ACT_TANH), torch.tanh(u).numpy(), rtol=1e-14, atol=1e-14)
    assert np.allclose(oracle_mod.features(x, A, oracle_mod.ACT_IDENTITY), u.numpy(), rtol=1e-14, atol=1e-14)
    # SiLU(0) = 0; its minimum sits where sigma(u)(1 + u(1 - sigma(u))) = 0, u* = -1.27846454...,
    # value -0.27846454... (u* = -(1 + e^u*)); probe it through a 1x1 projection
    one = np.ones((1, 1))
    assert oracle_mod.features(np.zeros((1, 1)), one, oracle_mod.ACT_SILU)[0, 0] == 0.0
    us = -1.2784645427610738
    assert abs(us + 1.0 + math.exp(us)) < 1e-15
    val = oracle_mod.features(np.full((1, 1), us), one, oracle_mod.ACT_SILU)[0, 0]
    assert abs(val - (1.0 + us)) < 1e-14  # at the minimum SiLU(u*) = 1 + u*
    grid = np.linspace(us - 0.5, us + 0.5, 101)[:, None]
    assert oracle_mod.features(grid, one, oracle_mod.ACT_SILU).min() >= val - 1e-15


@pytest.mark.parametrize("act", [1, 2, 3])
def test_lowrank_summary_equals_quadratic_other_activations(oracle_mod, act):
    """The summary form equals the explicit quadratic form for every activation (the summary's
    factorisation does not depend on the map).  Non-negative q, k and A keep the normaliser away
    from zero for identity and tanh."""
    w = W.TINY
    x = I.make_inputs(w)
    dec = oracle_mod.decode_bf16
    q, k, v = np.abs(dec(x["q"][0, :, 0])), np.abs(dec(x["k"][0, :, 0])), dec(x["v"][0, :, 0])
    A = np.abs(dec(x["A"]))
    r = oracle_mod.head_forward(q, k, v, A, (w.T, w.H, w.W), w.block, w.keep_frac, w.rank, branches=2,
                                activation=act)
    ref = brute.lowrank_quadratic(r["psiq"], r["phiq"], r["psik"], r["phik"], v)
    assert np.allclose(r["out_lowrank"], ref, rtol=1e-11, atol=1e-13)


def test_lowrank_without_rope(oracle_mod):
    """lowrank_rope=False (the no-RoPE ablation): psi = phi, so the branch is plain linear attention
    phi(q)^T sum_j phi(k_j) v_j / (phi(q) . sum_j phi(k_j) + 1e-6); it is then independent of the
    rotary base and of any position offset, and differs from the rotated branch."""
    w = W.TINY
    r0, x = _head(oracle_mod, w, branches=2, lowrank_rope=False)
    v = oracle_mod.decode_bf16(x["v"][0, :, 0])
    assert np.array_equal(r0["psiq"], r0["phiq"]) and np.array_equal(r0["psik"], r0["phik"])
    num = r0["phiq"] @ (r0["phik"].T @ v)
    den = r0["phiq"] @ r0["phik"].sum(0) + 1e-6
    assert np.allclose(r0["out_lowrank"], num / den[:, None], rtol=1e-11, atol=1e-13)
    r1, _ = _head(oracle_mod, w, branches=2, lowrank_rope=False, theta=500.0, offset=(3, 1, 2))
    assert np.allclose(r1["out_lowrank"], r0["out_lowrank"], rtol=1e-13, atol=1e-15)
    r2, _ = _head(oracle_mod, w, branches=2)
    assert not np.allclose(r2["out_lowrank"], r0["out_lowrank"], rtol=1e-3)


def test_full_width_linear_attention_baseline(oracle_mod):
    """r = D, A = I, relu, no low-rank RoPE: the branch is ReLU linear attention with a D x D
    context, out_i = relu(q_i) (relu(K)^T V) / (relu(q_i) . sum_j relu(k_j) + 1e-6) -- the full-width
    linear branch the pages compare against (RoPeSLR appendix FLOP analysis, RoLA App. F)."""
    w = W.TINY.with_(rank=64)
    x = I.make_inputs(w)
    dec = oracle_mod.decode_bf16
    q, k, v = dec(x["q"][0, :, 1]), dec(x["k"][0, :, 1]), dec(x["v"][0, :, 1])
    r = oracle_mod.head_forward(q, k, v, np.eye(64), (w.T, w.H, w.W), w.block, w.keep_frac, 64, branches=2,
                                lowrank_rope=False)
    fq, fk = np.maximum(q, 0), np.maximum(k, 0)
    ctx = fk.T @ v                      # D x D context, computed once per head
    ref = (fq @ ctx) / (fq @ fk.sum(0) + 1e-6)[:, None]
    assert np.allclose(r["out_lowrank"], ref, rtol=1e-12, atol=1e-14)


def test_lowrank_summary_equals_quadratic(oracle_mod):
    """The query-independent summary form (RoLA B.1) equals the explicit L x L quadratic form."""
    w = W.TINY
    r, x = _head(oracle_mod, w, branches=2)
    v = oracle_mod.decode_bf16(x["v"][0, :, 0])
    ref = brute.lowrank_quadratic(r["psiq"], r["phiq"], r["psik"], r["phik"], v)
    assert np.allclose(r["out_lowrank"], ref, rtol=1e-11, atol=1e-13)
    # the truncated rotation touches only the first r coordinates
    assert np.array_equal(r["psik"][:, w.rank:], r["phik"][:, w.rank:]) or r["psik"].shape[1] == w.rank


def test_lowrank_kernel_is_relative(oracle_mod):
    """psi(q_i) . psi(k_j) equals the relative-angle form (depends on p_i - p_j only), for the
    rank-truncated schedule (first r/2 pairs of the D-wide table) with r = 64 < D = 128 (spans the
    t and h axes)."""
    rng = np.random.default_rng(5)
    D, R, grid = 128, 64, (3, 4, 5)
    L = 60
    phiq = np.maximum(rng.standard_normal((L, R)), 0)
    phik = np.maximum(rng.standard_normal((L, R)), 0)
    psiq = oracle_mod.rope_rows(phiq, grid, R // 2, schedule_dim=D)
    psik = oracle_mod.rope_rows(phik, grid, R // 2, schedule_dim=D)
    axis, omega = oracle_mod.rope_pairs(D)
    pos = brute.grid_positions(grid)
    ref = brute.relative_kernel(phiq, phik, pos, pos, axis, omega, R // 2)
    assert np.allclose(psiq @ psik.T, ref, rtol=0, atol=1e-12)
    assert set(axis[:R // 2]) == {0, 1}  # 22 temporal pairs, then 10 height pairs


def test_lowrank_identity_projection_full_rank(oracle_mod):
    """r = D, A = I: features are relu(x) and the readout weight is relu(q)^T R(p_j - p_i) relu(k)."""
    rng = np.random.default_rng(6)
    D, grid = 64, (2, 3, 4)
    L = 24
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    r = oracle_mod.head_forward(q, k, v, np.eye(D), grid, 8, 1.0, D, branches=2)
    axis, omega = oracle_mod.rope_pairs(D)
    pos = brute.grid_positions(grid)
    wgt = brute.relative_kernel(np.maximum(q, 0), np.maximum(k, 0), pos, pos, axis, omega, D // 2)
    den = (np.maximum(q, 0) @ np.maximum(k, 0).T).sum(1, keepdims=True) + 1e-6
    assert np.allclose(r["out_lowrank"], (wgt @ v) / den, rtol=1e-10, atol=1e-12)


def test_lowrank_r32_rotates_temporal_pairs_only(oracle_mod):
    """r = 32 < 2 * 22: the truncated rotation uses temporal pairs only, so with one frame (T = 1)
    psi = phi exactly."""
    rng = np.random.default_rng(7)
    phi = np.maximum(rng.standard_normal((40, 32)), 0)
    psi = oracle_mod.rope_rows(phi, (1, 5, 8), 16, schedule_dim=128)
    assert np.array_equal(psi, phi)


# ------------------------------------------------------------------------------- whole forward
def test_forward_shift_invariant(oracle_mod):
    """Shifting all (t, h, w) positions by a constant leaves masks and both branches unchanged
    (RoPE relative invariance, RoLA eq. (1) and B.1)."""
    w = W.TINY
    x = I.make_inputs(w)
    g = (w.T, w.H, w.W)
    o0, p0 = oracle_mod.forward(x, g, w.block, w.keep_frac, w.rank)
    o1, p1 = oracle_mod.forward(x, g, w.block, w.keep_frac, w.rank, offset=(5, -3, 17))
    for key in p0:
        assert np.array_equal(p0[key]["idx"], p1[key]["idx"])
    assert np.allclose(o0, o1, rtol=0, atol=1e-11)


def test_forward_single_block_degenerate(oracle_mod):
    """L smaller than one block: one block, k = 1, the sparse branch is dense attention."""
    grid = (1, 3, 5)
    x = I.make_custom(12, 1, grid, 1, 64, 16)
    dec = oracle_mod.decode_bf16
    q, k, v, A = dec(x["q"][0, :, 0]), dec(x["k"][0, :, 0]), dec(x["v"][0, :, 0]), dec(x["A"])
    r = oracle_mod.head_forward(q, k, v, A, grid, 64, 0.1, 16)
    assert r["keep"] == 1 and r["idx"].tolist() == [[0]] and r["tie"][0] == 0
    ref = brute.masked_dense_attention(r["qh"], r["kh"], v, np.ones((15, 15), bool))
    assert np.allclose(r["out_sparse"], ref, rtol=0, atol=1e-12)
    assert np.allclose(r["out"], r["out_sparse"] + r["out_lowrank"], rtol=0, atol=0)


def test_forward_thread_count_independent(oracle_mod):
    """The oracle's results do not depend on the OpenMP thread count (fixed summation order)."""
    import subprocess, sys, json
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, hashlib; sys.path.insert(0, %r); import oracle;"
            "from sparse_rank_hybrid_b200 import workloads as W, inputs as I;"
            "w = W.TINY; x = I.make_inputs(w);"
            "o, _ = oracle.forward(x, (w.T, w.H, w.W), w.block, w.keep_frac, w.rank);"
            "print(hashlib.sha256(o.tobytes()).hexdigest())") % root
    outs = []
    for n in ("1", "4"):
        env = dict(os.environ, OMP_NUM_THREADS=n, PYTHONHASHSEED="0")
        outs.append(subprocess.check_output([sys.executable, "-c", code], env=env).strip())
    assert outs[0] == outs[1]


# --------------------------------------------------------------- pins catch planted mistakes
def test_pins_catch_planted_mistakes(oracle_mod):
    """Plant plausible mistakes into oracle outputs on the CPU and check the pins reject them."""
    rng = np.random.default_rng(8)
    D, grid = 64, (3, 4, 5)
    L = 60
    x = rng.standard_normal((L, D))
    axis, omega = oracle_mod.rope_pairs(D)
    pos = brute.grid_positions(grid)
    good = oracle_mod.rope_rows(x, grid, D // 2)
    assert np.allclose(good, brute.rope_complex(x, pos, axis, omega, D // 2), atol=1e-13)
    # (a) sin sign flipped (clockwise rotation)
    xs = x.copy(); xs[:, 1::2] *= -1
    bad = oracle_mod.rope_rows(xs, grid, D // 2); bad[:, 1::2] *= -1
    assert not np.allclose(bad, brute.rope_complex(x, pos, axis, omega, D // 2), atol=1e-6)
    # (b) axes swapped (h positions used for t pairs)
    pos_bad = pos[:, [1, 0, 2]]
    assert not np.allclose(good, brute.rope_complex(x, pos_bad, axis, omega, D // 2), atol=1e-6)
    # (c) normaliser with rotated instead of unrotated features
    phiq = np.maximum(rng.standard_normal((L, 16)), 0)
    phik = np.maximum(rng.standard_normal((L, 16)), 0)
    v = rng.standard_normal((L, D))
    psiq = oracle_mod.rope_rows(phiq, grid, 8, schedule_dim=D)
    psik = oracle_mod.rope_rows(phik, grid, 8, schedule_dim=D)
    S, z = oracle_mod.summary(psik, phik, v)
    good = oracle_mod.lowrank_apply(psiq, phiq, S, z)
    assert np.allclose(good, brute.lowrank_quadratic(psiq, phiq, psik, phik, v), rtol=1e-10)
    bad = oracle_mod.lowrank_apply(psiq, psiq, S, psik.sum(0))
    assert not np.allclose(bad, brute.lowrank_quadratic(psiq, phiq, psik, phik, v), rtol=1e-4)
    # (d) softmax scale dropped
    qh, kh = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    idx = np.arange(1)[None].repeat(1, 0)
    full = oracle_mod.sparse_attn(qh, kh, v, 64, idx)
    assert np.allclose(full, brute.masked_dense_attention(qh, kh, v, np.ones((L, L), bool)), atol=1e-12)
    unscaled = oracle_mod.sparse_attn(qh * math.sqrt(D), kh, v, 64, idx)
    assert not np.allclose(unscaled, brute.masked_dense_attention(qh, kh, v, np.ones((L, L), bool)),
                           atol=1e-4)


# ------------------------------------------------------------------- separate / per-head projections
def test_separate_projections_relative_form(oracle_mod):
    """Separate query and key projections Pq != Pk (RoLA E.2): the readout weight of query i on key j
    is relu(q_i Pq)^T R(p_j - p_i) relu(k_j Pk) over the first r coordinates, and the normaliser uses
    the unrotated features.  Both are written out here from numpy features and the brute relative
    kernel, so an oracle that swapped the projections or used one for both sides fails."""
    rng = np.random.default_rng(11)
    D, R, grid = 64, 32, (2, 3, 4)
    L = 24
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    Pq, Pk = rng.standard_normal((D, R)) / 8, rng.standard_normal((D, R)) / 8
    r = oracle_mod.head_forward(q, k, v, Pq, grid, 8, 1.0, R, branches=2, A_k=Pk)
    fq, fk = np.maximum(q @ Pq, 0), np.maximum(k @ Pk, 0)
    axis, omega = oracle_mod.rope_pairs(D)
    pos = brute.grid_positions(grid)
    wgt = brute.relative_kernel(fq, fk, pos, pos, axis, omega, R // 2)
    den = fq @ fk.sum(0) + 1e-6
    assert np.allclose(r["out_lowrank"], (wgt @ v) / den[:, None], rtol=1e-10, atol=1e-12)
    swapped = oracle_mod.head_forward(q, k, v, Pk, grid, 8, 1.0, R, branches=2, A_k=Pq)
    assert not np.allclose(swapped["out_lowrank"], r["out_lowrank"], rtol=1e-3)


def test_projection_layout_per_head_and_separate(oracle_mod):
    """forward() with per-head and/or separate projections reads head h's matrices from entry h,
    query side first: entries equal to the shared matrix reproduce the shared run exactly, a head whose
    entry is another matrix reproduces a shared run with that matrix, and Pq = A, Pk = B differs from
    both shared runs."""
    w = W.TINY
    x = I.make_inputs(w)
    grid = (w.T, w.H, w.W)
    other = I.make_projections(4242, 1, w.head_dim, w.rank, False, False)[0, 0]

    def run(A, **kw):
        y = dict(x)
        y["A"] = A
        return oracle_mod.forward(y, grid, w.block, w.keep_frac, w.rank, branches=2, **kw)[0]

    shared, shared_o = run(x["A"]), run(other)
    per_head = run(np.stack([x["A"], other])[None], proj_per_head=True)   # head 0: A, head 1: other
    assert np.array_equal(per_head[:, :, 0], shared[:, :, 0])
    assert np.array_equal(per_head[:, :, 1], shared_o[:, :, 1])
    same = run(np.stack([x["A"], x["A"]])[:, None], proj_separate=True)
    assert np.array_equal(same, shared)
    mixed = run(np.stack([x["A"], other])[:, None], proj_separate=True)  # Pq = A, Pk = other
    assert not np.allclose(mixed, shared, rtol=1e-3) and not np.allclose(mixed, shared_o, rtol=1e-3)
    both = run(np.stack([np.stack([x["A"], other]), np.stack([x["A"], other])]), proj_separate=True,
               proj_per_head=True)
    assert np.array_equal(both[:, :, 0], shared[:, :, 0]) and np.array_equal(both[:, :, 1], shared_o[:, :, 1])


# ------------------------------------------------------------------------------------ gated fusion
def _gated(oracle_mod, w_gate, b_gate, v_scale=1.0):
    w = W.TINY
    x = I.make_inputs(w)
    dec = oracle_mod.decode_bf16
    q, k, v = dec(x["q"][0, :, 0]), dec(x["k"][0, :, 0]), dec(x["v"][0, :, 0]) * v_scale
    r = oracle_mod.head_forward(q, k, v, dec(x["A"]), (w.T, w.H, w.W), w.block, w.keep_frac, w.rank,
                                gate=(np.asarray(w_gate, dtype=np.float64), b_gate))
    return r, q


def _rms(a):
    return np.sqrt((a ** 2).mean(axis=1))


def test_gate_closed_is_sparse_only(oracle_mod):
    """A very negative gate bias closes the gate: the output is the sparse branch alone, the
    module's starting point (RoLA 4.4)."""
    r, _ = _gated(oracle_mod, np.zeros(64), -1e4)
    assert np.array_equal(r["out"], r["out_sparse"])


def test_gate_half_open_adds_half_the_sparse_rms(oracle_mod):
    """w = 0, b = 0: the gate is 1/2 on every row, the added term points along the low-rank output
    and its RMS is half the sparse output's (the scale reference), up to the 1e-6 in the normaliser."""
    r, _ = _gated(oracle_mod, np.zeros(64), 0.0)
    add = r["out"] - r["out_sparse"]
    lr = r["out_lowrank"]
    eps_f = _rms(lr) / np.sqrt(_rms(lr) ** 2 + 1e-6)
    assert np.allclose(_rms(add), 0.5 * _rms(r["out_sparse"]) * eps_f, rtol=1e-10)
    cos = (add * lr).sum(1) / (np.linalg.norm(add, axis=1) * np.linalg.norm(lr, axis=1))
    assert np.allclose(cos, 1.0, atol=1e-12)


def test_gate_reads_the_raw_query(oracle_mod):
    """w = e_0, b = 0: the gate of row i, recovered from the RMS of the added term, is sigmoid(q_i[0])
    of the raw (pre-RoPE) query; the rotated query would give another value on rows with t > 0."""
    w_gate = np.zeros(64)
    w_gate[0] = 1.0
    r, q = _gated(oracle_mod, w_gate, 0.0)
    lr = r["out_lowrank"]
    unit = _rms(r["out_sparse"]) * _rms(lr) / np.sqrt(_rms(lr) ** 2 + 1e-6)
    g = _rms(r["out"] - r["out_sparse"]) / unit
    assert np.allclose(g, 1.0 / (1.0 + np.exp(-q[:, 0])), rtol=1e-9)
    assert not np.allclose(g, 1.0 / (1.0 + np.exp(-r["qh"][:, 0])), rtol=1e-3)


def test_gate_is_homogeneous_in_v(oracle_mod):
    """Both branches are linear in v and the RMS ratio does not change when v is scaled, so scaling v
    by 2 doubles the gated output, up to the 1e-6 in the RMS normaliser (here a relative effect of at
    most 1e-6 / (2 mean(O_lr^2)) ~ 3e-5 on the added term).  A scale reference that is not of degree
    one in v (say the mean square instead of the RMS) fails by a factor of 2."""
    rng = np.random.default_rng(3)
    w_gate = rng.standard_normal(64) / 8
    r1, _ = _gated(oracle_mod, w_gate, -1.0)
    r2, _ = _gated(oracle_mod, w_gate, -1.0, v_scale=2.0)
    ref = 2.0 * r1["out"]
    assert np.abs(r2["out"] - ref).max() <= 5e-5 * np.abs(ref).max()


# ----------------------------------------------------------------------- RoPE inside the activation
def _inside(oracle_mod, act=0, offset=(0, 0, 0), **kw):
    w = W.TINY
    x = I.make_inputs(w)
    dec = oracle_mod.decode_bf16
    q, k, v = dec(x["q"][0, :, 1]), dec(x["k"][0, :, 1]), dec(x["v"][0, :, 1])
    A = dec(x["A"])
    r = oracle_mod.head_forward(q, k, v, A, (w.T, w.H, w.W), w.block, w.keep_frac, w.rank, branches=2,
                                activation=act, offset=offset, **kw)
    return r, (q, k, v, A, w)


def test_rope_inside_written_out(oracle_mod):
    """RoPE inside the activation (RoLA 5.3 / B.3 ordering): psi = relu(R_r(p) (x A)) with the rotation
    done here by complex multiplication, and out = psi_q (psi_k^T v) / (psi_q . sum_j psi_k + 1e-6),
    both sides using the rotated-then-activated features."""
    r, (q, k, v, A, w) = _inside(oracle_mod, rope_inside=True)
    axis, omega = oracle_mod.rope_pairs(w.head_dim)
    pos = brute.grid_positions((w.T, w.H, w.W))
    pq = np.maximum(brute.rope_complex(q @ A, pos, axis, omega, w.rank // 2), 0)
    pk = np.maximum(brute.rope_complex(k @ A, pos, axis, omega, w.rank // 2), 0)
    ref = (pq @ (pk.T @ v)) / (pq @ pk.sum(0) + 1e-6)[:, None]
    assert np.allclose(r["out_lowrank"], ref, rtol=1e-10, atol=1e-12)


def test_rope_inside_identity_map_shares_the_numerator(oracle_mod):
    """With the identity map the rotation and the activation commute, so the inside and outside
    orderings give the same psi; only the normaliser differs (inside: rotated features)."""
    ri, _ = _inside(oracle_mod, act=2, rope_inside=True)
    ro, _ = _inside(oracle_mod, act=2)
    assert np.allclose(ri["psiq"], ro["psiq"], rtol=0, atol=1e-13)
    assert np.array_equal(ri["phiq"], ri["psiq"]) and not np.allclose(ri["phiq"], ro["phiq"], rtol=1e-3)


def test_rope_inside_is_not_shift_invariant(oracle_mod):
    """RoLA Table 2's contrast on synthetic features: shifting every position by a constant leaves the
    outside-activation branch unchanged (relative property) but changes the inside-activation one
    (absolute position leaks through the nonlinearity); without RoPE nothing changes."""
    def resid(**kw):
        a, _ = _inside(oracle_mod, **kw)
        b, _ = _inside(oracle_mod, offset=(2, 3, 5), **kw)
        return np.linalg.norm(a["out_lowrank"] - b["out_lowrank"]) / np.linalg.norm(a["out_lowrank"])
    assert resid() < 1e-12
    assert resid(lowrank_rope=False) == 0.0
    assert resid(rope_inside=True) > 1e-2


# ---------------------------------------------------------------------------------------- backward
def _bw_case(oracle_mod, keep_frac=0.5, seed=9):
    w = W.TINY.with_(keep_frac=keep_frac)
    x = I.make_inputs(w)
    dec = oracle_mod.decode_bf16
    q, k, v = dec(x["q"][0, :, 0]), dec(x["k"][0, :, 0]), dec(x["v"][0, :, 0])
    A = dec(x["A"])
    dout = np.random.default_rng(seed).standard_normal(q.shape)
    return w, q, k, v, A, dout


def test_backward_restatement_matches_forward(oracle_mod):
    """The differentiable fp64 torch restatement of the forward gives the C oracle's output."""
    from oracle import backward as B
    w, q, k, v, A, dout = _bw_case(oracle_mod)
    g = B.head_backward(q, k, v, A, dout, (w.T, w.H, w.W), w.block, w.keep_frac, w.rank)
    r = oracle_mod.head_forward(q, k, v, A, (w.T, w.H, w.W), w.block, w.keep_frac, w.rank)
    assert np.array_equal(g["idx"], r["idx"])
    assert np.allclose(g["out"], r["out"], rtol=1e-12, atol=1e-12)


def test_backward_matches_finite_differences(oracle_mod):
    """<grad, d> equals the central difference of sum(dout * out) along random directions d of q, k, v
    and A, the forward evaluated by the C oracle with the selection held fixed (both branches; the
    relu kinks are not crossed at this step size)."""
    from oracle import backward as B
    w, q, k, v, A, dout = _bw_case(oracle_mod)
    grid = (w.T, w.H, w.W)
    g = B.head_backward(q, k, v, A, dout, grid, w.block, w.keep_frac, w.rank)
    rng = np.random.default_rng(4)
    h = 1e-6

    def f(qq, kk, vv, AA):
        r = oracle_mod.head_forward(qq, kk, vv, AA, grid, w.block, w.keep_frac, w.rank, idx_override=g["idx"])
        return float((dout * r["out"]).sum())

    for name, arr in (("q", q), ("k", k), ("v", v), ("A", A)):
        d = rng.standard_normal(arr.shape)
        args = dict(qq=q, kk=k, vv=v, AA=A)
        key = {"q": "qq", "k": "kk", "v": "vv", "A": "AA"}[name]
        plus, minus = dict(args), dict(args)
        plus[key], minus[key] = arr + h * d, arr - h * d
        fd = (f(**plus) - f(**minus)) / (2 * h)
        an = float((g["d" + name] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_dense_sparse_branch_matches_sdpa(oracle_mod):
    """keep = 1, sparse branch only: the gradients equal torch's fp64 scaled-dot-product-attention
    backward on the rotated q, k, rotated back to the raw inputs (R(p)^T)."""
    import torch
    from oracle import backward as B
    w, q, k, v, A, dout = _bw_case(oracle_mod, keep_frac=1.0)
    grid = (w.T, w.H, w.W)
    g = B.head_backward(q, k, v, A, dout, grid, w.block, 1.0, w.rank, branches=1)
    qh = torch.tensor(oracle_mod.rope_rows(q, grid, w.head_dim // 2), requires_grad=True)
    kh = torch.tensor(oracle_mod.rope_rows(k, grid, w.head_dim // 2), requires_grad=True)
    vv = torch.tensor(v, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(qh[None, None], kh[None, None], vv[None, None])[0, 0]
    dqh, dkh, dv = torch.autograd.grad(o, (qh, kh, vv), torch.from_numpy(dout))
    cs = B.rope_cos_sin(grid, w.head_dim)

    def unrotate(y):  # R(p)^T y: rotate each pair by the negative angle
        y = y.numpy()
        x = y.copy()
        c, s = cs[:, :, 0], cs[:, :, 1]
        x[:, 0::2] = y[:, 0::2] * c + y[:, 1::2] * s
        x[:, 1::2] = -y[:, 0::2] * s + y[:, 1::2] * c
        return x

    assert np.allclose(g["dq"], unrotate(dqh), rtol=1e-10, atol=1e-12)
    assert np.allclose(g["dk"], unrotate(dkh), rtol=1e-10, atol=1e-12)
    assert np.allclose(g["dv"], dv.numpy(), rtol=1e-10, atol=1e-12)
    assert not g["dA"].any()


_BW_OPTIONS = [
    dict(activation=1, rope="inside", separate=True, gate=True),    # SiLU, RoPE inside, Pq != Pk, gated
    dict(activation=2, rope="none", separate=False, gate=False),    # identity map, no low-rank RoPE
    dict(activation=3, rope="outside", separate=True, gate=True),   # tanh, Pq != Pk, gated
]


def _bw_options_case(oracle_mod, opt):
    w, q, k, v, A, dout = _bw_case(oracle_mod)
    q, k, A = np.abs(q), np.abs(k), np.abs(A)   # non-negative features keep the normaliser conditioned
    rng = np.random.default_rng(21)
    Ak = np.abs(rng.standard_normal(A.shape)) / 8 if opt["separate"] else None
    gate = (rng.standard_normal(w.head_dim) / 8, -0.5) if opt["gate"] else None
    fwd = dict(activation=opt["activation"], lowrank_rope=opt["rope"] != "none", rope_inside=opt["rope"] == "inside",
               A_k=Ak, gate=gate)
    bwd = dict(activation=opt["activation"], rope=opt["rope"], A_k=Ak, gate=gate)
    return w, q, k, v, A, dout, Ak, gate, fwd, bwd


@pytest.mark.parametrize("opt", _BW_OPTIONS, ids=lambda o: f"act{o['activation']}-{o['rope']}-sep{o['separate']}-gate{o['gate']}")
def test_backward_options_restatement_and_finite_differences(oracle_mod, opt):
    """With the forward's options (feature map, RoPE ordering, separate key projection, gated fusion)
    the torch restatement reproduces the C oracle's forward, and its gradients -- including those of
    the key projection and of the gate's weights and bias -- match central differences of the C
    forward."""
    from oracle import backward as B
    w, q, k, v, A, dout, Ak, gate, fwd, bwd = _bw_options_case(oracle_mod, opt)
    grid = (w.T, w.H, w.W)
    g = B.head_backward(q, k, v, A, dout, grid, w.block, w.keep_frac, w.rank, **bwd)
    r = oracle_mod.head_forward(q, k, v, A, grid, w.block, w.keep_frac, w.rank, **fwd)
    assert np.allclose(g["out"], r["out"], rtol=1e-11, atol=1e-12)

    def f(qq=q, kk=k, vv=v, AA=A, AAk=Ak, gw=None, gb=None):
        kw = dict(fwd)
        kw["A_k"] = AAk
        if gate is not None:
            kw["gate"] = (gate[0] if gw is None else gw, gate[1] if gb is None else gb)
        rr = oracle_mod.head_forward(qq, kk, vv, AA, grid, w.block, w.keep_frac, w.rank, idx_override=g["idx"], **kw)
        return float((dout * rr["out"]).sum())

    rng = np.random.default_rng(5)
    h = 1e-6
    cases = [("dq", "qq", q), ("dk", "kk", k), ("dv", "vv", v), ("dA", "AA", A)]
    if Ak is not None:
        cases.append(("dA_k", "AAk", Ak))
    if gate is not None:
        cases.append(("dgate_w", "gw", gate[0]))
    for name, key, arr in cases:
        d = rng.standard_normal(np.shape(arr))
        fd = (f(**{key: arr + h * d}) - f(**{key: arr - h * d})) / (2 * h)
        an = float((g[name] * d).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
    if gate is not None:
        fd = (f(gb=gate[1] + h) - f(gb=gate[1] - h)) / (2 * h)
        assert abs(fd - float(g["dgate_b"])) <= 1e-6 * max(1.0, abs(fd)), ("dgate_b", fd, float(g["dgate_b"]))


def test_backward_steps_match_autograd(oracle_mod):
    """The explicit gradient steps (flash-style sparse backward with lse and Delta; the low-rank chain
    through the summary, the normaliser, R_r^T, the relu mask and A^T) give autograd's gradients: the
    derivation the GPU backward is to follow."""
    from oracle import backward as B
    for keep in (0.5, 1.0):
        w, q, k, v, A, dout = _bw_case(oracle_mod, keep_frac=keep)
        grid = (w.T, w.H, w.W)
        g = B.head_backward(q, k, v, A, dout, grid, w.block, keep, w.rank)
        m = B.head_backward_steps(q, k, v, A, dout, grid, w.block, w.rank, g["idx"])
        for name in ("dq", "dk", "dv", "dA"):
            assert np.allclose(m[name], g[name], rtol=1e-10, atol=1e-12), name


def test_backward_sampled_equals_full_steps(oracle_mod):
    """head_backward_sampled (the gradients evaluated only on chosen query / key blocks, plus dA, for
    full-size heads) equals head_backward_steps on every block of a small ragged case, for a subset of
    blocks, and for empty subsets (dA alone); a key block that no query block kept gets only its
    low-rank gradient."""
    from oracle import backward as OB
    rng = np.random.default_rng(31)
    grid, D, R, block = (3, 5, 7), 32, 16, 16  # L = 105: a ragged last block of 9 tokens
    L = 105
    q, k, v = (rng.standard_normal((L, D)) for _ in range(3))
    A = rng.standard_normal((D, R)) / np.sqrt(D)
    dout = rng.standard_normal((L, D))
    qh, kh = oracle_mod.rope_rows(q, grid, D // 2), oracle_mod.rope_rows(k, grid, D // 2)
    s = oracle_mod.block_scores(oracle_mod.block_means(qh, block), oracle_mod.block_means(kh, block))
    nb = s.shape[0]
    idx, _ = oracle_mod.topk(s, 2)
    full = OB.head_backward_steps(q, k, v, A, dout, grid, block, R, idx)
    rows = lambda a: slice(a * block, min(L, (a + 1) * block))
    for qbs, kbs in ((range(nb), range(nb)), ([0, nb - 1], [3, nb - 1]), ([], [])):
        smp = OB.head_backward_sampled(q, k, v, A, dout, grid, block, R, idx, qbs, kbs)
        assert np.allclose(smp["dA"], full["dA"], rtol=1e-12, atol=1e-12)
        for a in qbs:
            assert np.allclose(smp["dq"][a], full["dq"][rows(a)], rtol=1e-12, atol=1e-12)
        for b in kbs:
            assert np.allclose(smp["dk"][b], full["dk"][rows(b)], rtol=1e-12, atol=1e-12)
            assert np.allclose(smp["dv"][b], full["dv"][rows(b)], rtol=1e-12, atol=1e-12)
