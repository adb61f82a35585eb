"""Host-side checks of the seeded input generator and of the benchmark's option handling (CPU only):
the projection and gate draws have the documented shapes and seeds and leave the q/k/v draws alone,
and each benchmark flag reaches the oracle and the library problem as intended."""
import argparse

import numpy as np

import bench
from sparse_rank_hybrid_b200 import inputs as I
from sparse_rank_hybrid_b200 import workloads as W


def _args(**kw):
    base = dict(activation="relu", lowrank_norope=False, linear_baseline=False, branches="both", proj="shared",
                fusion="sum", rope_inside=False)
    base.update(kw)
    return argparse.Namespace(**base)


def test_projection_draws():
    w = W.TINY
    for sep, ph in ((0, 0), (1, 0), (0, 1), (1, 1)):
        a = I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, bool(sep), bool(ph))
        assert a.dtype == np.uint16 and a.shape == (1 + sep, w.heads if ph else 1, w.head_dim, w.rank)
        b = I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, bool(sep), bool(ph))
        assert np.array_equal(a, b)
    # entries are distinct draws, roughly N(0, 1/D)
    a = I.bf16_bits_to_f32(I.make_projections(7, 4, 128, 32, True, True)).astype(np.float64)
    assert not np.array_equal(a[0, 0], a[1, 0]) and not np.array_equal(a[0, 0], a[0, 1])
    assert abs(a.std() - 1 / np.sqrt(128)) < 0.01


def test_run_inputs_follow_the_flags():
    w = W.TINY
    base = I.make_inputs(w)
    x = bench.make_run_inputs(_args(), w)
    assert all(np.array_equal(x[n], base[n]) for n in ("q", "k", "v", "A"))
    x = bench.make_run_inputs(_args(proj="separate-per-head"), w)
    assert x["A"].shape == (2, w.heads, w.head_dim, w.rank)
    assert all(np.array_equal(x[n], base[n]) for n in ("q", "k", "v"))   # q, k, v unchanged
    x = bench.make_run_inputs(_args(linear_baseline=True), w.with_(rank=w.head_dim))
    assert np.array_equal(x["A"], np.eye(w.head_dim, dtype=np.uint16) * 0x3F80)


def test_variant_keywords():
    w = W.TINY
    v = bench.variant_of(_args(activation="silu", lowrank_norope=True, branches="lowrank"), w)
    assert v["activation"] == 1 and v["lowrank_rope"] is False and v["branches"] == 2 and v["gate"] is None
    v = bench.variant_of(_args(proj="separate", fusion="gated", rope_inside=True), w)
    assert v["proj_separate"] and not v["proj_per_head"] and v["rope_inside"]
    wg, bg = v["gate"]
    assert wg.shape == (w.head_dim,) and bg == bench.GATE_BIAS < 0
    assert np.array_equal(wg, bench.gate_weights(w).astype(np.float64))
