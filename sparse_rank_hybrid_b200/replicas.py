"""Host-side logic for running the forward pass as independent replicas, one process per GPU.

Every (batch, head) problem of the method is independent (selection, low-rank summary and attention
are all per head), so several GPUs need no data-path exchange: each rank runs its own problem and
only the timing is combined (slowest rank's device time, total work of all ranks).  The collectives
here carry timing scalars only, over whatever process group is initialised (NCCL on GPUs, gloo in
the CPU tests).
"""
from __future__ import annotations

from .workloads import Workload


def replica_workload(w: Workload, rank: int) -> Workload:
    """Rank 0 runs the workload itself; rank r > 0 an independent problem of the same shape (its own
    seeds), so per-GPU work is fixed as ranks are added (weak scaling)."""
    if rank == 0:
        return w
    a_seed = None if w.a_seed is None else w.a_seed + 7919 * rank
    return w.with_(name=f"{w.name}#r{rank}", seed=w.seed + 7919 * rank, a_seed=a_seed)


def _reduce(x: float, op_name: str, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return float(t.item())


def max_over_ranks(x: float, device=None) -> float:
    """Slowest rank's value (device times are combined this way, never by wall clock)."""
    return _reduce(x, "MAX", device)


def sum_over_ranks(x: float, device=None) -> float:
    return _reduce(x, "SUM", device)


def job_throughput(total_flops: float, max_ms: float) -> float:
    """Whole-job TFLOP/s: all ranks' work over the slowest rank's time."""
    return total_flops / (max_ms * 1e-3) / 1e12
