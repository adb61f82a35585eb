"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol that
include/slra.h declares, and validates problems / sizes workspaces without touching a device."""
import os
import re
import subprocess

import numpy as np
import pytest

from sparse_rank_hybrid_b200 import build as B
from sparse_rank_hybrid_b200 import slra
from sparse_rank_hybrid_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def _declared():
    src = open(os.path.join(ROOT, "include", "slra.h")).read()
    return sorted(set(re.findall(r"\b(slra_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    out = subprocess.check_output(["nm", "-D", "--defined-only", B.LIB], text=True)
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    declared = _declared()
    assert set(declared) == set(slra.EXPORTS)
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    # nothing else leaks out of the library (internal C++ symbols are hidden)
    assert {s for s in exported if s.startswith("slra_")} == set(declared)


def test_abi_version_and_status_strings():
    assert slra.lib().slra_abi_version() == slra.ABI_VERSION == 8
    for s in range(0, 9):
        assert slra.status_string(s) and slra.status_string(s) != "unknown status"
    assert slra.status_string(99) == "unknown status"


@pytest.mark.parametrize("w", list(W.MAIN.values()), ids=lambda w: w.name)
def test_keep_count_and_layout(w, oracle_mod):
    p = slra.Problem.from_workload(w)
    assert slra.validate(p) == slra.OK
    assert slra.keep_count(p) == oracle_mod.keep_count(w.keep_frac, w.nb)
    lay = slra.layout(p)
    assert lay.nb == w.nb and lay.L == w.L
    offs = sorted(lay.offsets.values())
    assert all(o % 256 == 0 for o in offs) and offs[0] == 0 and lay.total_bytes >= offs[-1]


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, slra.ERR_UNSUPPORTED), ("block", 32, slra.ERR_UNSUPPORTED),
    ("rank", 24, slra.ERR_UNSUPPORTED), ("rank", 256, slra.ERR_UNSUPPORTED), ("rank", 0, slra.ERR_UNSUPPORTED),
    ("keep_frac", 0.0, slra.ERR_INVALID_ARG), ("keep_frac", 1.5, slra.ERR_INVALID_ARG),
    ("T", 0, slra.ERR_INVALID_ARG), ("heads", 0, slra.ERR_INVALID_ARG), ("out_dtype", 7, slra.ERR_INVALID_ARG),
    ("rope_split", (10, 10, 10), slra.ERR_INVALID_ARG), ("branches", 9, slra.ERR_INVALID_ARG),
    ("T", 5000, slra.ERR_UNSUPPORTED),  # 5000*45*80 tokens -> more than 2048 blocks
    ("activation", 4, slra.ERR_INVALID_ARG), ("activation", -1, slra.ERR_INVALID_ARG),
    ("lowrank_norope", 2, slra.ERR_INVALID_ARG),
    ("proj_separate", 2, slra.ERR_INVALID_ARG), ("proj_per_head", -1, slra.ERR_INVALID_ARG),
    ("fusion", 2, slra.ERR_INVALID_ARG), ("fusion", slra.FUSION_GATED, slra.ERR_INVALID_ARG),  # no gate_w
    ("lowrank_rope_inside", 2, slra.ERR_INVALID_ARG),
])
def test_validation_rejects(field, value, status):
    p = slra.Problem.from_workload(W.WAN_14B)
    setattr(p, field, value)
    assert slra.validate(p) == status


@pytest.mark.parametrize("separate,per_head", [(0, 0), (1, 0), (0, 1), (1, 1)])
def test_projection_elems_and_layout(separate, per_head):
    """The projection argument holds (1 + separate) x (per_head ? heads : 1) matrices of D x rank;
    per-head projections give the workspace one readout image per head (head_dim 128), and the
    intermediates keep their offsets."""
    w = W.WAN_14B
    p = slra.Problem.from_workload(w, proj_separate=separate, proj_per_head=per_head)
    n = (1 + separate) * (w.heads if per_head else 1) * w.head_dim * w.rank
    assert slra.projection_elems(p) == n == int(np.prod(p.projection_shape))
    base = slra.layout(slra.Problem.from_workload(w))
    lay = slra.layout(p)
    assert lay.offsets == base.offsets
    extra = (w.heads - 1) * w.rank * 256 if per_head else 0
    assert base.total_bytes + extra <= lay.total_bytes <= base.total_bytes + extra + 256
    assert slra.projection_elems(slra.Problem.from_workload(w, proj_separate=3)) == -1


@pytest.mark.parametrize("gate_w,branches,bias,status", [
    (4096, 3, -2.0, slra.OK), (4096, 0, 0.5, slra.OK), (4100, 3, -2.0, slra.ERR_ALIGNMENT),
    (4096, 1, -2.0, slra.ERR_INVALID_ARG), (4096, 2, -2.0, slra.ERR_INVALID_ARG),
    (4096, 3, float("nan"), slra.ERR_INVALID_ARG), (4096, 3, float("inf"), slra.ERR_INVALID_ARG),
])
def test_gated_fusion_validation(gate_w, branches, bias, status):
    """The gated fusion needs its weight vector (16-B aligned device pointer; validation never
    dereferences it), a finite bias and both branches."""
    import ctypes
    p = slra.Problem.from_workload(W.TINY).c()
    p.fusion, p.gate_w, p.branches, p.gate_bias = slra.FUSION_GATED, gate_w, branches, bias
    assert slra.lib().slra_validate(ctypes.byref(p)) == status


def test_rope_inside_excludes_norope():
    p = slra.Problem.from_workload(W.TINY, lowrank_rope_inside=1)
    assert slra.validate(p) == slra.OK
    p.lowrank_norope = 1
    assert slra.validate(p) == slra.ERR_INVALID_ARG


def test_host_pipeline_plan():
    """The host entry point pipelines about sixteen head groups per batch element when two group slots
    fit the buffers it is given, and falls back to one group otherwise (no GPU needed)."""
    def groups(w, io=None, ws=None, **kw):
        p = slra.Problem.from_workload(w, **kw)
        return slra.host_pipeline_groups(p, slra.host_io_bytes(p) if io is None else io,
                                         slra.layout(p).total_bytes if ws is None else ws)
    assert groups(W.WAN_14B) == 14 and groups(W.WAN_1_3B) == 12   # 40 heads in groups of 3; 12 of 1
    assert groups(W.WAN_14B, proj_separate=1, proj_per_head=1) == 14
    assert groups(W.TINY) == 1                      # two one-head slots need more than the 2-head workspace
    assert groups(W.WAN_14B, io=1 << 20) == 1 and groups(W.WAN_14B, ws=1 << 20) == 1
    bad = slra.Problem.from_workload(W.WAN_14B.with_(rank=24))
    assert slra.host_pipeline_groups(bad, 1 << 40, 1 << 40) == -1


def test_validation_grid_limit():
    """batch x heads is a launch grid dimension (at most 65535); a tiny sequence keeps every other
    limit far away, so only that one decides."""
    p = slra.Problem.from_workload(W.TINY)
    p.heads = 65535
    assert slra.validate(p) == slra.OK
    p.heads = 65536
    assert slra.validate(p) == slra.ERR_UNSUPPORTED


def test_calls_without_device_fail_cleanly():
    """On a machine without a GPU every compute entry point returns an error status (never crashes)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    p = slra.Problem.from_workload(W.TINY)
    lay = slra.layout(p)
    import ctypes
    buf = ctypes.create_string_buffer(lay.total_bytes + 512)
    base = (ctypes.addressof(buf) + 255) // 256 * 256
    s = slra.lib().slra_attn_fwd_ex(ctypes.byref(p.c()), base, base, base, base, base + 256, base, lay.total_bytes,
                                    None)
    assert s != slra.OK
    # descriptor-style entry points: well-formed, disjoint host pointers reach the device check
    n = W.TINY.batch * W.TINY.L * W.TINY.heads * W.TINY.head_dim
    bufs = [ctypes.create_string_buffer(n * 4 + 256) for _ in range(4)]
    ptrs = [(ctypes.addressof(b) + 255) // 256 * 256 for b in bufs]
    t = [slra._Tensor(ptrs[i], slra.DTYPE_BF16, 1, W.TINY.L, W.TINY.heads, W.TINY.head_dim, 0, 0, 0) for i in range(3)]
    o = slra._Tensor(ptrs[3], slra.DTYPE_F32, 1, W.TINY.L, W.TINY.heads, W.TINY.head_dim, 0, 0, 0)
    a_buf = ctypes.create_string_buffer(64 * 16 * 2 + 256)
    a = slra._Mat((ctypes.addressof(a_buf) + 255) // 256 * 256, slra.DTYPE_BF16, 64, 16)
    args = (4, 8, 8)
    assert slra.lib().slra_attn_fwd(*(ctypes.byref(x) for x in t), ctypes.byref(a), *args, 64, 0.5, 16,
                                    ctypes.byref(o), None) == slra.ERR_NO_DEVICE
    assert slra.lib().slra_sparse_fwd(*(ctypes.byref(x) for x in t), *args, 64, 0.5, ctypes.byref(o), None, 0,
                                      None) == slra.ERR_NO_DEVICE
    assert slra.lib().slra_lowrank_fwd(*(ctypes.byref(x) for x in t), ctypes.byref(a), *args, 16, ctypes.byref(o),
                                       None, None, None, 0, None) == slra.ERR_NO_DEVICE
    st = ctypes.c_int32(-1)
    assert slra.lib().slra_get_device_status(None, ctypes.byref(st)) == slra.ERR_NO_DEVICE
    # invalid descriptors are rejected before the device is looked at
    bad_L = slra._Tensor(ptrs[0], slra.DTYPE_BF16, 1, W.TINY.L + 1, W.TINY.heads, W.TINY.head_dim, 0, 0, 0)
    assert slra.lib().slra_attn_fwd(ctypes.byref(bad_L), ctypes.byref(t[1]), ctypes.byref(t[2]), ctypes.byref(a),
                                    *args, 64, 0.5, 16, ctypes.byref(o), None) == slra.ERR_INVALID_ARG
    f32_q = slra._Tensor(ptrs[0], slra.DTYPE_F32, 1, W.TINY.L, W.TINY.heads, W.TINY.head_dim, 0, 0, 0)
    assert slra.lib().slra_attn_fwd(ctypes.byref(f32_q), ctypes.byref(t[1]), ctypes.byref(t[2]), ctypes.byref(a),
                                    *args, 64, 0.5, 16, ctypes.byref(o), None) == slra.ERR_INVALID_ARG
    a_rank = slra._Mat(a.data, slra.DTYPE_BF16, 64, 32)
    assert slra.lib().slra_attn_fwd(*(ctypes.byref(x) for x in t), ctypes.byref(a_rank), *args, 64, 0.5, 16,
                                    ctypes.byref(o), None) == slra.ERR_INVALID_ARG
    alias = slra._Tensor(ptrs[0], slra.DTYPE_F32, 1, W.TINY.L, W.TINY.heads, W.TINY.head_dim, 0, 0, 0)
    assert slra.lib().slra_attn_fwd(*(ctypes.byref(x) for x in t), ctypes.byref(a), *args, 64, 0.5, 16,
                                    ctypes.byref(alias), None) == slra.ERR_INVALID_ARG


def test_workspace_bytes_matches_layout():
    for w in (W.TINY, W.WAN_1_3B, W.WAN_14B, W.HUNYUAN):
        assert slra.workspace_bytes(w.batch, w.heads, w.head_dim, w.T, w.H, w.W, w.block, w.keep_frac, w.rank) == \
            slra.layout(slra.Problem.from_workload(w)).total_bytes
    assert slra.workspace_bytes(1, 2, 96, 4, 8, 8, 64, 0.5, 16) == 0  # head_dim 96 is not supported


@pytest.mark.parametrize("field,value,status", [
    ("q_strides", (0, 0, 0), slra.OK),
    ("q_strides", None, slra.OK),                       # fused QKV: [B][L][3][Hh][D] views
    ("k_strides", "headmajor", slra.OK),                # [B][Hh][L][D] input
    ("v_strides", (8, 8, 8), slra.OK),                  # inputs may alias (read only)
    ("q_strides", (0, 0, 4), slra.ERR_INVALID_ARG),     # not a multiple of 8 elements
    ("q_strides", (0, 512, 64), slra.ERR_INVALID_ARG),  # zero stride with others set
    ("out_strides", (0, 0, 0), slra.OK),
    ("out_strides", "headmajor", slra.OK),
    ("out_strides", "padded", slra.OK),                 # rows padded to 96 fp32
    ("out_strides", (8, 8, 8), slra.ERR_INVALID_ARG),   # output rows overlap
    ("out_strides", "shortrow", slra.ERR_INVALID_ARG),  # head stride below D: rows overlap
])
def test_stride_validation(field, value, status):
    w = W.TINY
    L, Hh, D = w.L, w.heads, w.head_dim
    spec = {None: (L * 3 * Hh * D, 3 * Hh * D, D), "headmajor": (Hh * L * D, D, L * D),
            "padded": (L * Hh * 96, Hh * 96, 96), "shortrow": (L * Hh * 32, Hh * 32, 32)}
    p = slra.Problem.from_workload(w, **{field: spec.get(value, value) if not isinstance(value, tuple) else value})
    assert slra.validate(p) == status


def test_host_entry_point_rejects_strides():
    import ctypes
    p = slra.Problem.from_workload(W.TINY, q_strides=(W.TINY.L * 3 * 128, 3 * 128, 64))
    assert slra.validate(p) == slra.OK
    b = ctypes.create_string_buffer(1 << 20)
    base = (ctypes.addressof(b) + 255) // 256 * 256
    s = slra.lib().slra_attn_fwd_host(ctypes.byref(p.c()), base, base, base, base, base, base, 1 << 19, base,
                                      1 << 19, None)
    assert s == slra.ERR_INVALID_ARG


def args_g(*a):
    return a


def test_train_forward_and_saved_backward_validation():
    """slra_attn_fwd_train wants a backward-sized workspace and the backward's options; both new entry
    points check their arguments before looking for a device."""
    import ctypes
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    p = slra.Problem.from_workload(W.TINY)
    n = W.TINY.batch * W.TINY.L * W.TINY.heads * W.TINY.head_dim
    bufs = [ctypes.create_string_buffer(n * 4 + 256) for _ in range(9)]
    q, k, v, A, out, dout, dq, dk, dv = [(ctypes.addressof(b) + 255) // 256 * 256 for b in bufs]
    dA_buf = ctypes.create_string_buffer(64 * 16 * 4 + 256)
    dA = (ctypes.addressof(dA_buf) + 255) // 256 * 256
    fwd_b = slra.layout(p).total_bytes
    bwd_b = slra.bwd_workspace_bytes(p)
    assert bwd_b > fwd_b
    ws_buf = ctypes.create_string_buffer(bwd_b + 256)
    ws = (ctypes.addressof(ws_buf) + 255) // 256 * 256
    L = slra.lib()
    pc = p.c()
    # a forward-sized workspace is too small for the kept state; NULL is not allowed
    assert L.slra_attn_fwd_train(ctypes.byref(pc), q, k, v, A, out, ws, fwd_b, None) == slra.ERR_WORKSPACE
    assert L.slra_attn_fwd_train(ctypes.byref(pc), q, k, v, A, out, None, 0, None) == slra.ERR_WORKSPACE
    assert L.slra_attn_fwd_train(ctypes.byref(pc), q, k, v, A, out, ws + 16, bwd_b, None) == slra.ERR_WORKSPACE
    assert L.slra_attn_fwd_train(ctypes.byref(pc), q, k, v, A, out, ws, bwd_b, None) == slra.ERR_NO_DEVICE
    # options the backward does not cover are refused by the training forward too
    # the gated fusion: covered too (its backward also wants the gate gradients' outputs)
    pg = slra.Problem.from_workload(W.TINY).c()
    pg.fusion = slra.FUSION_GATED
    pg.gate_w = dA
    bwd_g = L.slra_bwd_workspace_bytes(ctypes.byref(pg))
    assert bwd_g > bwd_b  # O_lr, dO_lr and the gate's partial sums
    gbuf = ctypes.create_string_buffer(bwd_g + 256)
    gws = (ctypes.addressof(gbuf) + 255) // 256 * 256
    assert L.slra_attn_fwd_train(ctypes.byref(pg), q, k, v, A, out, gws, bwd_g, None) == slra.ERR_NO_DEVICE
    assert L.slra_attn_bwd(ctypes.byref(pg), *args_g(q, k, v, A, dout, dq, dk, dv, dA), gws, bwd_g,
                           None) == slra.ERR_INVALID_ARG  # no dgate_w / dgate_b
    gw_buf = ctypes.create_string_buffer(64 * 4 + 256 + 16)
    pg.dgate_w = (ctypes.addressof(gw_buf) + 255) // 256 * 256
    pg.dgate_b = pg.dgate_w + 64 * 4
    assert L.slra_attn_bwd(ctypes.byref(pg), *args_g(q, k, v, A, dout, dq, dk, dv, dA), gws, bwd_g,
                           None) == slra.ERR_NO_DEVICE
    pg.dgate_b = pg.dgate_w + 8  # overlaps dgate_w
    assert L.slra_attn_bwd(ctypes.byref(pg), *args_g(q, k, v, A, dout, dq, dk, dv, dA), gws, bwd_g,
                           None) == slra.ERR_INVALID_ARG
    # the feature maps, RoPE orderings and projection layouts are covered: they reach the device check
    for field, value in (("activation", slra.ACT_SILU), ("lowrank_rope_inside", 1), ("lowrank_norope", 1)):
        po = slra.Problem.from_workload(W.TINY).c()
        setattr(po, field, value)
        assert L.slra_attn_fwd_train(ctypes.byref(po), q, k, v, A, out, ws, bwd_b, None) == slra.ERR_NO_DEVICE
    # the saved backward: same checks as slra_attn_bwd
    args = (q, k, v, A, dout, dq, dk, dv, dA)
    assert L.slra_attn_bwd_saved(ctypes.byref(pc), *args, ws, bwd_b - 256, None) == slra.ERR_WORKSPACE
    assert L.slra_attn_bwd_saved(ctypes.byref(pc), *args, ws, bwd_b, None) == slra.ERR_NO_DEVICE
    assert L.slra_attn_bwd_saved(ctypes.byref(pc), q, k, v, A, dout, dq, dq, dv, dA, ws, bwd_b,
                                 None) == slra.ERR_INVALID_ARG


def test_backward_rejects_strided_outputs():
    """The gradients are contiguous: a problem with output strides is refused by the backward entry
    points (before any device access), while the forward accepts it."""
    import ctypes
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    p = slra.Problem.from_workload(W.TINY)
    pc = p.c()
    D, Hh = W.TINY.head_dim, W.TINY.heads
    pc.out_strides[:] = [W.TINY.L * Hh * D * 2, Hh * D * 2, D]  # rows of a wider buffer
    assert slra.lib().slra_bwd_workspace_bytes(ctypes.byref(pc)) == 0
    assert slra.lib().slra_validate(ctypes.byref(pc)) == slra.OK
