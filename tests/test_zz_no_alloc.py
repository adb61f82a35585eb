"""The allocation-free low-rank summary (slra_lowrank_summary_noalloc) against the workspace one.

The entry point is for callers that cannot allocate device memory where they call it (a host
framework that owns all device memory through its own pool, an execute hook that must not allocate,
a serving loop that cannot afford cudaMalloc's device-wide synchronization).  It keeps its scratch
in one fixed array inside the library, so this test checks that two calls in a row, on different
problem sizes, each reproduce slra_lowrank_summary within the summary tolerance, i.e. that nothing a
previous call left in the shared array leaks into the next result, and that a bounded wait that
runs out inside the summary kernel is reported through slra_noalloc_device_status instead of
passing silently.

This file is collected last so that a failure here cannot hide another test's result.
"""
import numpy as np
import pytest

from sparse_rank_hybrid_b200 import inputs as I
from sparse_rank_hybrid_b200 import slra
from sparse_rank_hybrid_b200 import workloads as W

pytestmark = pytest.mark.gpu

SUMMARY_REL = 1e-4  # same bound as the summary parity tests


@pytest.fixture(scope="module", autouse=True)
def _build():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_rank_hybrid_b200 import build
    build.build()


def _gpu(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _both(w):
    import torch
    p = slra.Problem.from_workload(w)
    x = I.make_inputs(w)
    k, v, A = _gpu(x["k"]), _gpu(x["v"]), _gpu(x["A"])
    ws = slra.lowrank_summary(p, k, v, A)
    S_ref = slra.ws_view(p, ws, "S").clone()
    z_ref = slra.ws_view(p, ws, "z").clone()
    BH = w.batch * w.heads
    S = torch.full((BH, w.rank, w.head_dim), float("nan"), dtype=torch.float32, device="cuda")
    z = torch.full((BH, w.rank), float("nan"), dtype=torch.float32, device="cuda")
    slra.lowrank_summary_noalloc(p, k, v, A, S, z)
    torch.cuda.synchronize()
    return S, z, S_ref, z_ref


def _rel(a, b):
    return float((a - b).norm() / b.norm())


def test_noalloc_summary_matches_workspace_entry_point_twice():
    # first a larger problem (many splits, rank 64), then a smaller one that reuses the same scratch
    for w in (W.WAN_1_3B.with_(rank=64, heads=6), W.TINY):
        S, z, S_ref, z_ref = _both(w)
        assert bool(S.isfinite().all()) and bool(z.isfinite().all()), w.name
        assert _rel(S, S_ref) < SUMMARY_REL, (w.name, _rel(S, S_ref))
        assert _rel(z, z_ref) < SUMMARY_REL, (w.name, _rel(z, z_ref))


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 320 heads x rank 128 x (128 + 1) fp32 partial sums (21 MB) do not fit the 16 MiB area even unsplit
    p = slra.Problem(1, 320, 128, 4, 8, 8, 128, 0.1, 128)
    import torch
    k = torch.zeros((1, p.L, 320, 128), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    S = torch.empty((320, 128, 128), dtype=torch.float32, device="cuda")
    z = torch.empty((320, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(slra.SlraError) as e:
        slra.lowrank_summary_noalloc(p, k, k, A, S, z)
    assert e.value.status == slra.ERR_SCRATCH_LIMIT


# head_dim 128 (the tensor-core summary kernel, whose waits are bounded), L = 390 with a ragged tile
EDGE_128 = W.Workload("noalloc-edge-128", 1, 2, 128, 3, 10, 13, 32, 128, 0.3, 7160)


def test_noalloc_reports_a_timeout_and_recovers():
    """The test hook makes every summary CTA wait on a barrier nothing signals; the wait runs out after
    1 ms, the kernel records a timeout and returns, and the call's status reader reports it (once: it
    clears the word).  The next call starts from a cleared status word and matches the workspace entry
    point again."""
    import torch
    w = EDGE_128
    x = I.make_inputs(w)
    k, v, A = _gpu(x["k"]), _gpu(x["v"]), _gpu(x["A"])
    BH = w.batch * w.heads
    S = torch.zeros((BH, w.rank, w.head_dim), dtype=torch.float32, device="cuda")
    z = torch.zeros((BH, w.rank), dtype=torch.float32, device="cuda")
    p_hang = slra.Problem.from_workload(w, debug_flags=slra.DEBUG_UNSATISFIED_WAIT, wait_timeout_ns=1_000_000)
    slra.lowrank_summary_noalloc(p_hang, k, v, A, S, z)
    assert slra.noalloc_device_status() == slra.ERR_DEVICE_TIMEOUT
    assert slra.noalloc_device_status() == slra.OK
    S2, z2, S_ref, z_ref = _both(w)
    assert slra.noalloc_device_status() == slra.OK
    assert _rel(S2, S_ref) < SUMMARY_REL and _rel(z2, z_ref) < SUMMARY_REL
