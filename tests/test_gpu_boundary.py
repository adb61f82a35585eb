"""The C-ABI boundary on the GPU: the descriptor-style entry points and strided tensors.

  - slra_attn_fwd (tensor descriptors, library-allocated workspace) gives slra_attn_fwd_ex's output
    bit for bit: both run the same kernels on the same bytes;
  - q, k, v as strided views (one fused QKV buffer, or head-major [B][Hh][L][D] storage) and a padded
    output give the contiguous call's output bit for bit (the kernels read rows through strided tensor
    maps; nothing is copied);
  - slra_sparse_fwd and slra_lowrank_fwd give the branch-restricted slra_attn_fwd_ex output bit for bit,
    the latter also its S and z;
  - a NULL workspace (stream-ordered allocation inside the library) gives the caller-workspace output
    bit for bit and reports its device status through slra_get_device_status;
  - the fp16 v copy in the workspace is written by the selection-only call and the training forward
    (for the backward kernels) and left alone by the inference forward, which reads v itself;
and the descriptor call is checked against the oracle once.  Inputs: the seeded generator.
"""
import numpy as np
import pytest

from sparse_rank_hybrid_b200 import inputs as I
from sparse_rank_hybrid_b200 import slra
from sparse_rank_hybrid_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

EDGE_128 = W.Workload("boundary-edge-128", 2, 3, 128, 3, 10, 13, 32, 64, 0.3, 7620)  # batch 2, ragged


@pytest.fixture(scope="module", autouse=True)
def _build():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_rank_hybrid_b200 import build
    build.build()
    import oracle
    oracle.build()


def _inputs(w):
    x = I.make_inputs(w)
    return x, {n: parity.to_gpu(x[n]) for n in ("q", "k", "v", "A")}


def _ex(w, t, **kw):
    p = slra.Problem.from_workload(w, **kw)
    out, ws = slra.attn_fwd(p, t["q"], t["k"], t["v"], t["A"] if p.branches & slra.BRANCH_LOWRANK else None)
    assert slra.device_status(ws) == slra.OK
    return out, ws, p


@pytest.mark.parametrize("w", [W.TINY, EDGE_128], ids=lambda w: w.name)
def test_descriptor_call_equals_problem_call(w):
    import torch
    x, t = _inputs(w)
    ref, _, _ = _ex(w, t)
    out = torch.empty_like(ref)
    slra.attn_fwd_tensors(t["q"], t["k"], t["v"], t["A"], w.T, w.H, w.W, w.block, w.keep_frac, w.rank, out)
    assert slra.get_device_status() == slra.OK
    assert torch.equal(out, ref)
    parity.compare(slra.Problem.from_workload(w), x, {"out": out.double().cpu().numpy()},
                   label=f"{w.name}-descriptors")


@pytest.mark.parametrize("w", [W.TINY, EDGE_128], ids=lambda w: w.name)
@pytest.mark.parametrize("layout", ["fused-qkv", "head-major", "padded-out"])
def test_strided_tensors_equal_contiguous(w, layout):
    import torch
    _, t = _inputs(w)
    ref, _, _ = _ex(w, t)
    B, L, Hh, D = ref.shape
    if layout == "fused-qkv":
        qkv = torch.stack([t["q"], t["k"], t["v"]], dim=2).contiguous()  # [B, L, 3, Hh, D]
        q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
        out = torch.empty_like(ref)
    elif layout == "head-major":
        q, k, v = (t[n].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3) for n in ("q", "k", "v"))
        out = torch.empty((B, Hh, L, D), dtype=ref.dtype, device=ref.device).permute(0, 2, 1, 3)
    else:
        q, k, v = t["q"], t["k"], t["v"]
        out = torch.full((B, L, Hh, D + 32), float("nan"), dtype=ref.dtype, device=ref.device)[..., :D]
    assert not (q.is_contiguous() and out.is_contiguous())
    p = slra.Problem.from_workload(w)
    got, ws = slra.attn_fwd(p, q, k, v, t["A"], out=out)
    assert slra.device_status(ws) == slra.OK
    assert torch.equal(got, ref)
    if layout == "padded-out":  # the padding columns are left alone
        assert bool(torch.isnan(out.as_strided((B, L, Hh, 32), out.stride(), out.storage_offset() + D)).all())
    # the descriptor-style call takes the same strided views
    got2 = torch.empty_like(out) if layout != "padded-out" else out
    slra.attn_fwd_tensors(q, k, v, t["A"], w.T, w.H, w.W, w.block, w.keep_frac, w.rank, got2)
    assert torch.equal(got2, ref)


@pytest.mark.parametrize("w", [W.TINY, EDGE_128], ids=lambda w: w.name)
def test_branch_entry_points(w):
    import torch
    x, t = _inputs(w)
    ref_s, _, _ = _ex(w, t, branches=slra.BRANCH_SPARSE)
    out = torch.empty_like(ref_s)
    slra.sparse_fwd(t["q"], t["k"], t["v"], w.T, w.H, w.W, w.block, w.keep_frac, out)
    assert slra.get_device_status() == slra.OK
    assert torch.equal(out, ref_s)
    ws = torch.empty(slra.workspace_bytes(w.batch, w.heads, w.head_dim, w.T, w.H, w.W, w.block, w.keep_frac, 16),
                     dtype=torch.uint8, device="cuda")
    out2 = torch.empty_like(ref_s)
    slra.sparse_fwd(t["q"], t["k"], t["v"], w.T, w.H, w.W, w.block, w.keep_frac, out2, workspace=ws)
    assert torch.equal(out2, ref_s)

    p_lr = slra.Problem.from_workload(w, branches=slra.BRANCH_LOWRANK)
    ref_l, ws_l = slra.attn_fwd(p_lr, t["q"], t["k"], t["v"], t["A"])
    BH = w.batch * w.heads
    S = torch.empty((BH, w.rank, w.head_dim), dtype=torch.float32, device="cuda")
    z = torch.empty((BH, w.rank), dtype=torch.float32, device="cuda")
    out3 = torch.empty_like(ref_l)
    slra.lowrank_fwd(t["q"], t["k"], t["v"], t["A"], w.T, w.H, w.W, w.rank, out3, S=S, z=z)
    assert slra.get_device_status() == slra.OK
    # the low-rank branch does not depend on the block size, so the call's output equals this one's
    assert torch.equal(out3, ref_l)
    assert torch.equal(S, slra.ws_view(p_lr, ws_l, "S")) and torch.equal(z, slra.ws_view(p_lr, ws_l, "z"))
    parity.compare(p_lr, x, {"out": out3.double().cpu().numpy()}, label=f"{w.name}-lowrank-entry")


def test_null_workspace_equals_caller_workspace():
    import torch
    w = EDGE_128
    _, t = _inputs(w)
    ref, _, p = _ex(w, t)
    got, ws = slra.attn_fwd(p, t["q"], t["k"], t["v"], t["A"], alloc_workspace_in_library=True)
    assert ws is None
    assert slra.get_device_status() == slra.OK
    assert torch.equal(got, ref)


def test_null_workspace_reports_device_status():
    """A device-side problem of a call whose workspace the library allocated (and freed) is still
    reported: here an input too large for the fp16 operands."""
    import torch
    w = W.TINY
    _, t = _inputs(w)
    q = t["q"].clone()
    q[0, 5, 0, 3] = 1e6
    out = torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32, device="cuda")
    slra.attn_fwd_tensors(q, t["k"], t["v"], t["A"], w.T, w.H, w.W, w.block, w.keep_frac, w.rank, out)
    assert slra.get_device_status() == slra.ERR_RANGE
    assert slra.get_device_status() == slra.OK


@pytest.mark.parametrize("w", [W.TINY, EDGE_128], ids=lambda w: w.name)
def test_overlapped_preparation_equals_serial(w):
    """With both branches on, the low-rank preparation runs on the library's side stream while the
    calling stream runs RoPE + pooling and selection; the result equals the serialised order bit for bit
    (the same kernels on the same bytes), also when two host threads call on two streams at once."""
    import threading
    import torch
    _, t = _inputs(w)
    ser, _, _ = _ex(w, t, debug_flags=slra.DEBUG_SERIAL_BRANCHES)
    ovl, _, _ = _ex(w, t)
    assert torch.equal(ser, ovl)
    p = slra.Problem.from_workload(w)
    outs, errs = [None, None], []

    def run(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                o, ws = slra.attn_fwd(p, t["q"], t["k"], t["v"], t["A"], stream=s)
                s.synchronize()
                assert slra.device_status(ws, stream=s) == slra.OK
                outs[i] = o
        except Exception as e:  # noqa: BLE001
            errs.append(e)

    th = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for x in th:
        x.start()
    for x in th:
        x.join()
    assert not errs, errs
    assert torch.equal(outs[0], ser) and torch.equal(outs[1], ser)


@pytest.mark.parametrize("w", [W.TINY, EDGE_128], ids=lambda w: w.name)
def test_v_copy_only_where_the_backward_reads_it(w):
    """The inference forward reads v from the caller's tensor and leaves the workspace's fp16 v section
    as it was; the selection-only call and the training forward write it (v in head-major order, rounded
    to fp16, zero padded to whole blocks) for the backward kernels, as the header's workspace layout
    states."""
    import torch
    _, t = _inputs(w)
    p = slra.Problem.from_workload(w)
    BH, Lp = w.batch * w.heads, w.nb * w.block
    expect = torch.zeros((BH, Lp, w.head_dim), dtype=torch.float16, device="cuda")
    expect[:, :w.L] = t["v"].permute(0, 2, 1, 3).reshape(BH, w.L, w.head_dim).half()

    ws = slra.alloc_workspace(p)
    slra.ws_view(p, ws, "vh").fill_(7.0)
    slra.attn_fwd(p, t["q"], t["k"], t["v"], t["A"], workspace=ws)
    assert slra.device_status(ws) == slra.OK
    assert torch.all(slra.ws_view(p, ws, "vh") == 7.0)
    slra.select_blocks(p, t["q"], t["k"], t["v"], workspace=ws)
    assert slra.device_status(ws) == slra.OK
    assert torch.equal(slra.ws_view(p, ws, "vh"), expect)

    wst = torch.empty(slra.bwd_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    slra.ws_view(p, wst, "vh").fill_(7.0)
    slra.attn_fwd_train(p, t["q"], t["k"], t["v"], t["A"], workspace=wst)
    assert slra.device_status(wst) == slra.OK
    assert torch.equal(slra.ws_view(p, wst, "vh"), expect)
