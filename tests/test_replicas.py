"""Multi-rank (replica) path of the benchmark on CPU: two gloo ranks combine timings and work the way
bench.py does on GPUs (max of device times, sum of work), with no data-path collective."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from sparse_rank_hybrid_b200 import replicas
from sparse_rank_hybrid_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 17.25][rank]
        local_flops = [1.0e12, 1.5e12][rank]
        mx = replicas.max_over_ranks(local_ms)
        tot = replicas.sum_over_ranks(local_flops)
        w = replicas.replica_workload(W.WAN_14B, rank)
        results[rank] = (mx, tot, w.seed, w.L, w.heads)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_combine_timing_and_work():
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(2, port, results), nprocs=2, join=True)
        r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 17.25                      # max over ranks
    assert r0[1] == r1[1] == 2.5e12                     # total work
    assert r0[2] == W.WAN_14B.seed and r1[2] != r0[2]   # rank 0 = the workload, rank 1 independent
    assert r0[3:] == r1[3:] == (W.WAN_14B.L, W.WAN_14B.heads)
    assert replicas.job_throughput(2.5e12, 17.25) == pytest.approx(2.5e12 / 17.25e-3 / 1e12)


def test_single_process_reductions_are_identity():
    assert replicas.max_over_ranks(3.0) == 3.0
    assert replicas.sum_over_ranks(4.0) == 4.0
    assert replicas.replica_workload(W.TINY, 0) is W.TINY
