#!/usr/bin/env python
"""Benchmark of the 3D-RoPE sparse + low-rank hybrid attention forward on B200.

One step = one full forward call (3D RoPE + pooling + top-k selection, low-rank summary, block-sparse
attention with the fused low-rank readout) over the Wan2.1-14B 720p shape: 75,600 tokens, 40 heads of
width 128, rank 32, 128-token blocks, 10% of key blocks kept (90% sparsity).  Inputs are the seeded
clustered-Gaussian bf16 tensors of `sparse_rank_hybrid_b200.inputs` (synthetic stand-ins for the real
activations), resident in HBM before timing; the L2 is flushed between timed steps.

Prints one JSON line (rank 0).  `value` is the effective TFLOP/s of the whole job (kept sparse FLOPs
+ low-rank FLOPs + block-score FLOPs, counted exactly from the selected masks, summed over ranks,
divided by the slowest rank's device time); `ms_per_step` is ms per attention call.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With --gpus N > 1 (under torchrun) every rank runs its own independent problem (a replica: the method
has no cross-head or cross-sample exchange), so per-GPU work is fixed and scaling is weak.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_rank_hybrid_b200 import flops as F  # noqa: E402
from sparse_rank_hybrid_b200 import inputs as I  # noqa: E402
from sparse_rank_hybrid_b200 import replicas  # noqa: E402
from sparse_rank_hybrid_b200 import workloads as WL  # noqa: E402

METRIC = "ms/attn call & effective TFLOP/s at L=75600, 40 heads, 90% sparsity; %roofline"
DEFAULT_WORKLOAD = WL.WAN_14B.name


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------- CPU oracle
ACTS = {"relu": 0, "silu": 1, "identity": 2, "tanh": 3}
BRANCHES = {"both": 3, "sparse": 1, "lowrank": 2}
# projection layouts: (separate Pq / Pk, one per head)
PROJS = {"shared": (0, 0), "separate": (1, 0), "per-head": (0, 1), "separate-per-head": (1, 1)}


def identity_bits(D: int) -> np.ndarray:
    """A = I as bf16 bits (1.0 = 0x3F80): the full-width linear-attention baseline's projection."""
    a = np.zeros((D, D), dtype=np.uint16)
    a[np.arange(D), np.arange(D)] = 0x3F80
    return a


GATE_BIAS = -2.0  # negative: the gated fusion starts near the sparse output (RoLA 4.4)


def gate_weights(w) -> np.ndarray:
    """Synthetic gate weights Wg ~ N(0, 1/head_dim), fp32, from the workload seed + 6000."""
    rng = np.random.default_rng(w.seed + 6000)
    return (rng.standard_normal(w.head_dim) / np.sqrt(w.head_dim)).astype(np.float32)


def variant_of(args, w) -> dict:
    """Low-rank branch and fusion options of the run (the oracle's keyword names)."""
    sep, ph = PROJS[args.proj]
    gate = (gate_weights(w).astype(np.float64), GATE_BIAS) if args.fusion == "gated" else None
    return {"activation": ACTS[args.activation], "lowrank_rope": not args.lowrank_norope,
            "branches": BRANCHES[args.branches], "proj_separate": bool(sep), "proj_per_head": bool(ph),
            "gate": gate, "rope_inside": bool(args.rope_inside)}


def make_run_inputs(args, w) -> dict:
    """The run's seeded inputs: the workload's q, k, v and A, with A replaced for the linear baseline
    (A = I) or a separate / per-head projection layout."""
    x = I.make_inputs(w)
    if args.linear_baseline:
        x["A"] = identity_bits(w.head_dim)
    elif args.proj != "shared":
        sep, ph = PROJS[args.proj]
        x["A"] = I.make_projections(w.seed + 5000, w.heads, w.head_dim, w.rank, bool(sep), bool(ph))
    return x


def oracle_sample(w, x, variant: dict, seconds_hint: float = 15.0):
    """Time the fp64 oracle on a bounded sample: one head's full selection and low-rank summary plus as
    many query blocks (attention + readout) as fit the hint.  Returns (tflops, desc, threads, secs)."""
    import oracle
    oracle.build()
    grid = (w.T, w.H, w.W)
    nb = w.nb
    threads = int(os.environ.get("OMP_NUM_THREADS", 0)) or len(os.sched_getaffinity(0))
    # a first call with one query block measures the per-block cost
    t0 = time.perf_counter()
    _, per = oracle.forward(x, grid, w.block, w.keep_frac, w.rank, heads=[(0, 0)], qblocks=[0], **variant)
    t1 = time.perf_counter()
    base = t1 - t0
    nq = 1
    if base < seconds_hint:
        # second call: more blocks to fill the budget (selection/low-rank cost repeats once)
        per_block = max(base / 4, 1e-3)
        nq = int(min(nb, max(2, (seconds_hint - base) / per_block)))
        qbs = list(np.linspace(0, nb - 1, nq).astype(int))
        t0 = time.perf_counter()
        _, per = oracle.forward(x, grid, w.block, w.keep_frac, w.rank, heads=[(0, 0)], qblocks=qbs, **variant)
        t1 = time.perf_counter()
    else:
        qbs = [0]
    secs = t1 - t0
    r = per[(0, 0)]
    sz = F.block_sizes(w.L, w.block)
    br = variant.get("branches", 3)
    kept = float(4.0 * w.head_dim * sum(sz[r["idx"][a]].sum() * sz[a] for a in qbs)) if br & 1 else 0.0
    rows = int(sum(sz[a] for a in qbs))
    work = kept + (F.score_flops(nb, w.head_dim, 1) if br & 1 else 0.0) + \
        ((4.0 * w.L * w.rank * w.head_dim + 4.0 * rows * w.rank * w.head_dim) if br & 2 else 0.0)
    desc = (f"fp64 C oracle, head (0,0) of {w.name}: full 3D RoPE, pooling, scores, top-k and low-rank "
            f"summary over all {w.L} tokens, plus attention + low-rank readout for {len(qbs)} of {nb} query "
            f"blocks; value = that work's effective FLOPs / wall time")
    return work / secs / 1e12, desc, threads, secs


def run_reference(args, w, rank, world):
    """Reference arm: the CPU oracle timed step by step on a bounded sample of the workload."""
    if rank != 0:
        return
    x = make_run_inputs(args, w)
    import oracle
    oracle.build()
    grid = (w.T, w.H, w.W)
    threads = len(os.sched_getaffinity(0))
    qbs = [0, w.nb - 1]

    def step():
        t0 = time.perf_counter()
        _, per = oracle.forward(x, grid, w.block, w.keep_frac, w.rank, heads=[(0, 0)], qblocks=qbs,
                                **variant_of(args, w))
        return time.perf_counter() - t0, per[(0, 0)]

    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t, r = step()
        times.append(t)
    sz = F.block_sizes(w.L, w.block)
    br = BRANCHES[args.branches]
    kept = float(4.0 * w.head_dim * sum(sz[r["idx"][a]].sum() * sz[a] for a in qbs)) if br & 1 else 0.0
    rows = int(sum(sz[a] for a in qbs))
    work = kept + (F.score_flops(w.nb, w.head_dim, 1) if br & 1 else 0.0) + \
        ((4.0 * w.L * w.rank * w.head_dim + 4.0 * rows * w.rank * w.head_dim) if br & 2 else 0.0)
    tot = sum(times)
    value = work * args.steps / tot / 1e12
    sample = (f"one step = head (0,0) of {w.name}: full selection and low-rank summary over {w.L} tokens "
              f"plus attention + readout for query blocks {qbs}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded clustered-Gaussian bf16 q/k/v, A ~ N(0, 1/d_h))",
            "config": {"workload": w.name, "L": w.L, "heads": w.heads, "head_dim": w.head_dim, "rank": w.rank,
                       "block": w.block, "keep_frac": w.keep_frac, "activation": args.activation,
                       "lowrank_rope": not args.lowrank_norope, "branches": args.branches,
                       "linear_baseline": bool(args.linear_baseline), "projection": args.proj,
                       "fusion": args.fusion, "rope_inside": bool(args.rope_inside)},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------- GPU arm
def _problem(args, w, slra, dev, torch, stage_ev):
    """The run's problem description and its seeded inputs on the device."""
    x = make_run_inputs(args, w)
    q, k, v = (torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    var = variant_of(args, w)
    gate_kw = {}
    if args.fusion == "gated":
        gate_kw = dict(fusion=slra.FUSION_GATED, gate_bias=GATE_BIAS,
                       gate_w=torch.from_numpy(gate_weights(w)).to(dev))
    prob = slra.Problem.from_workload(w, stage_events=tuple(e.cuda_event for e in stage_ev),
                                      branches=BRANCHES[args.branches], activation=var["activation"],
                                      lowrank_norope=int(not var["lowrank_rope"]),
                                      proj_separate=int(var["proj_separate"]), proj_per_head=int(var["proj_per_head"]),
                                      lowrank_rope_inside=int(args.rope_inside), **gate_kw)
    A = torch.from_numpy(x["A"].view(np.int16)).view(torch.bfloat16).to(dev).reshape(prob.projection_shape)
    return x, var, prob, (q, k, v, A)


def _work(w, prob, ws, slra, br):
    """Algorithmic FLOPs of one call, counted exactly from the selected masks: (total, sparse kept,
    low-rank, scores, attention kernel's own = kept + the fused readout's q A and psi S, keep)."""
    BH = w.batch * w.heads
    if br & 1:
        idx = slra.ws_view(prob, ws, "idx").cpu().numpy()
        f_sparse = F.sparse_flops(idx, w.L, w.block, w.head_dim)
        f_sc = F.score_flops(w.nb, w.head_dim, BH)
        keep_blocks = int(idx.shape[-1])
    else:
        f_sparse = f_sc = 0.0
        keep_blocks = 0
    f_lr = F.lowrank_flops(w.L, w.rank, w.head_dim, BH) if br & 2 else 0.0
    f_attn = f_sparse + (4.0 * w.L * w.rank * w.head_dim * BH if br & 2 else 0.0)
    return f_sparse + f_lr + f_sc, f_sparse, f_lr, f_sc, f_attn, keep_blocks


STAGES = ("rope_table", "rope_pool", "select", "lowrank_partial", "lowrank_reduce", "attention")


def _timed_calls(slra, torch, prob, tensors, out, ws, stage_ev, steps, warmup, flush, stream, barrier=lambda: None):
    """Warm up, then time `steps` calls with CUDA events on the launching stream, the L2 flushed before
    each.  Returns (per-call ms list, per-stage ms lists)."""
    q, k, v, A = tensors
    for _ in range(max(3, warmup)):
        slra.attn_fwd(prob, q, k, v, A, out=out, workspace=ws)
    torch.cuda.synchronize()
    status = slra.device_status(ws)
    if status != slra.OK:
        raise RuntimeError(f"device status after warm-up: {slra.status_string(status)}")
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    stage_ms = []
    barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        step_ev[i][0].record(stream)
        slra.attn_fwd(prob, q, k, v, A, out=out, workspace=ws)
        step_ev[i][1].record(stream)
        torch.cuda.synchronize()
        stage_ms.append([stage_ev[j].elapsed_time(stage_ev[j + 1]) for j in range(6)])
    barrier()
    torch.cuda.synchronize()
    status = slra.device_status(ws)
    if status != slra.OK:
        raise RuntimeError(f"device status after timing: {slra.status_string(status)}")
    return [a.elapsed_time(b) for a, b in step_ev], stage_ms


def _rooflines(w, f_sparse, f_attn, attn_ms, ms_per_step):
    """The attention kernel's roofline (its algorithmic FLOPs per launch / its event time, against the
    measured burst bf16 peak: the kernel is timed alone inside a step of a few ms) and the whole call's
    (max(kept FLOPs / tensor peak, minimum bytes / HBM bandwidth) against ms per call)."""
    hbm, tf_burst, tf_sust, src = peaks()
    achieved = f_attn / (attn_ms * 1e-3) / 1e12
    bytes_min = F.io_bytes(w.batch, w.L, w.heads, w.head_dim, w.rank, 4)
    t_roof = max(f_sparse / (tf_burst * 1e12), bytes_min / (hbm * 1e9))
    t_roof_sust = max(f_sparse / (tf_sust * 1e12), bytes_min / (hbm * 1e9))
    roof = {"kernel": "attn_sm100_kernel", "bound": "tensor", "achieved": achieved, "peak": tf_burst,
            "unit": "TFLOP/s", "frac": achieved / tf_burst,
            "peak_source": f"{src} burst bf16 (same rate as f16)", "attn_ms": attn_ms,
            "peak_sustained": tf_sust, "frac_of_sustained": achieved / tf_sust}
    call = {"t_roof_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_per_step,
            "frac_of_sustained": t_roof_sust * 1e3 / ms_per_step,
            "note": "max(kept FLOPs / burst tensor peak, min bytes / HBM peak) vs ms_per_step"}
    return roof, call


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from sparse_rank_hybrid_b200 import build as B
    from sparse_rank_hybrid_b200 import slra

    B.build()
    if rank == 0:
        import oracle
        oracle.build()  # compile the CPU baseline before any GPU work
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    base_w = w
    w = replicas.replica_workload(base_w, rank)  # each rank: its own independent problem
    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
    for e in stage_ev:
        e.record()
    torch.cuda.synchronize()
    x, var, prob, tensors = _problem(args, w, slra, dev, torch, stage_ev)
    br = BRANCHES[args.branches]
    ws = slra.alloc_workspace(prob, dev)
    out = torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32, device=dev)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    q, k, v, A = tensors
    slra.attn_fwd(prob, q, k, v, A, out=out, workspace=ws)
    torch.cuda.synchronize()
    f_total, f_sparse, f_lr, f_sc, f_attn, keep_blocks = _work(w, prob, ws, slra, br)

    clocks = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    clocks.start()
    time.sleep(0.3)
    step_ms, stage_ms = _timed_calls(slra, torch, prob, tensors, out, ws, stage_ev, args.steps, args.warmup, flush,
                                     stream, barrier)
    clk = clocks.stop()
    # per-kernel times: a few more calls with the branches' preparation serialised (the timed calls
    # overlap the low-rank preparation with RoPE + pooling and selection on a side stream)
    import dataclasses
    _, stage_serial = _timed_calls(slra, torch, dataclasses.replace(prob, debug_flags=slra.DEBUG_SERIAL_BRANCHES),
                                   tensors, out, ws, stage_ev, 3, 3, flush, stream)
    tot_ms = replicas.max_over_ranks(sum(step_ms), dev)
    ms_per_step = tot_ms / args.steps
    job_flops = replicas.sum_over_ranks(f_total, dev)

    # ---- end to end through the host entry point (pinned host buffers, copies inside the timing)
    host = {n: torch.from_numpy(x[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v", "A")}
    out_h = torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32).pin_memory()
    io = torch.empty(slra.host_io_bytes(prob), dtype=torch.uint8, device=dev)
    del flush
    slra.attn_fwd_host(prob, host["q"], host["k"], host["v"], host["A"], out_h, io, ws)
    e2e_steps = max(2, min(args.steps, 5))
    e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    barrier()
    for i in range(e2e_steps):
        e_ev[i][0].record(stream)
        slra.attn_fwd_host(prob, host["q"], host["k"], host["v"], host["A"], out_h, io, ws)
        e_ev[i][1].record(stream)
        torch.cuda.synchronize()
    e2e_ms = replicas.max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ev) / e2e_steps, dev)
    h2d = sum(int(host[n].numel()) * 2 for n in ("q", "k", "v", "A"))
    d2h = int(out_h.numel()) * 4

    if rank != 0:
        return
    stage_avg = [statistics.mean(x[i] for x in stage_ms) for i in range(6)]
    serial_avg = [statistics.mean(x[i] for x in stage_serial) for i in range(6)]
    roof, call_roof = _rooflines(w, f_sparse, f_attn, stage_avg[5], ms_per_step)
    roof["traffic"] = load_traffic(w.name)
    cpu_v, cpu_desc, cpu_threads, _ = oracle_sample(w, x, var)  # rank 0 runs the workload itself
    line = {
        "metric": METRIC, "value": replicas.job_throughput(job_flops, ms_per_step), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16 (S = q^k^T) and bf16 (P.V) tensor-core operands, fp32 accumulate, fp64 selection",
        "data": "synthetic (seeded clustered-Gaussian bf16 q/k/v, A ~ N(0, 1/d_h)); inputs resident in HBM",
        "config": {"workload": base_w.name, "L": w.L, "heads": w.heads, "head_dim": w.head_dim, "rank": w.rank,
                   "block": w.block, "keep_frac": w.keep_frac, "keep_blocks": keep_blocks,
                   "out_dtype": "f32", "l2": "flushed between timed steps (512 MB write)",
                   "parallelism": f"replica x{world} (independent problems, no collective)",
                   "activation": args.activation, "lowrank_rope": not args.lowrank_norope,
                   "branches": args.branches, "linear_baseline": bool(args.linear_baseline),
                   "projection": args.proj, "fusion": args.fusion, "rope_inside": bool(args.rope_inside)},
        "flops_per_step": {"sparse_kept": f_sparse, "lowrank": f_lr, "scores": f_sc},
        "roofline": roof,
        "call_roofline": call_roof,
        "e2e": {"value": replicas.job_throughput(job_flops, e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "stage_ms": {"rope_table": round(stage_avg[0], 4),
                     "preparation (rope_pool + select on the stream, low-rank summary on a side stream)":
                         round(sum(stage_avg[1:5]), 4), "attention": round(stage_avg[5], 4)},
        "kernel_ms": dict(zip(STAGES, (round(x, 4) for x in serial_avg))),
        "kernel_ms_note": "each kernel alone: 3 extra calls with the preparation serialised",
        "gpu_launches": 6 * args.steps,
        "clocks": clk,
        "cpu_baseline": {"value": cpu_v, "unit": "TFLOP/s", "cores": cpu_threads, "kind": "oracle",
                         "sample": cpu_desc},
    }
    print(json.dumps(line), flush=True)


def run_backward(args, w):
    """The backward pass (slra_attn_bwd) at the workload's shape on one GPU: ms per call, per-stage
    times, and the sparse gradient kernels' throughput against the algorithmic count (five products per
    kept (query block, key block) pair: S, dP, dQ, dK, dV = 2.5x the forward's kept FLOPs; the kernels
    recompute S and dP once more, which is not counted); then a training step, the forward that keeps
    its state followed by the backward from it.  One JSON line (not the benchmark contract)."""
    import torch
    from sparse_rank_hybrid_b200 import build as B
    from sparse_rank_hybrid_b200 import slra

    B.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    import dataclasses
    # the run's options (feature map, RoPE ordering, projections, gated fusion) as for the forward
    x, var, prob, (q, k, v, A) = _problem(args, w, slra, dev, torch, ev)
    dout = torch.from_numpy(I.make_dout(w.seed + 9000, w.batch, w.L, w.heads, w.head_dim)).to(dev)
    if prob.fusion == slra.FUSION_GATED:
        prob = dataclasses.replace(prob, dgate_w=torch.empty(w.head_dim, dtype=torch.float32, device=dev),
                                   dgate_b=torch.empty(1, dtype=torch.float32, device=dev))
    grads = tuple(torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32, device=dev)
                  for _ in range(3)) + (torch.empty(prob.projection_shape, dtype=torch.float32, device=dev),)
    ws = torch.empty(slra.bwd_workspace_bytes(prob), dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        slra.attn_bwd(prob, q, k, v, A, dout, grads=grads, workspace=ws)
    torch.cuda.synchronize()
    if slra.device_status(ws) != slra.OK:
        raise RuntimeError("device status after warm-up")
    f_total, f_sparse, f_lr, f_sc, f_attn, keep_blocks = _work(w, prob, ws, slra, 3)
    clocks = ClockSampler(0 if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[0]))
    clocks.start()
    time.sleep(0.3)
    tot, stages = [], []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        slra.attn_bwd(prob, q, k, v, A, dout, grads=grads, workspace=ws)
        b.record(stream)
        torch.cuda.synchronize()
        tot.append(a.elapsed_time(b))
        stages.append([ev[i].elapsed_time(ev[i + 1]) for i in range(6)])
    # A training step: the forward that keeps its state (slra_attn_fwd_train), then the backward from it
    # (slra_attn_bwd_saved), with no recompute.
    prob_f = dataclasses.replace(prob, stage_events=(None,) * 7)
    out = torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32, device=dev)
    for _ in range(max(3, args.warmup)):
        slra.attn_fwd_train(prob_f, q, k, v, A, out=out, workspace=ws)
        slra.attn_bwd_saved(prob, q, k, v, A, dout, ws, grads=grads)
    torch.cuda.synchronize()
    if slra.device_status(ws) != slra.OK:
        raise RuntimeError("device status after the training-step warm-up")
    t_fwd, t_bwd, st_saved = [], [], []
    for _ in range(args.steps):
        flush.zero_()
        a, m, b = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        slra.attn_fwd_train(prob_f, q, k, v, A, out=out, workspace=ws)
        m.record(stream)
        slra.attn_bwd_saved(prob, q, k, v, A, dout, ws, grads=grads)
        b.record(stream)
        torch.cuda.synchronize()
        t_fwd.append(a.elapsed_time(m))
        t_bwd.append(m.elapsed_time(b))
        st_saved.append([ev[i].elapsed_time(ev[i + 1]) for i in range(6)])
    clk = clocks.stop()
    if slra.device_status(ws) != slra.OK:
        raise RuntimeError("device status after timing")
    st = [statistics.mean(s_[i] for s_ in stages) for i in range(6)]
    sts = [statistics.mean(s_[i] for s_ in st_saved) for i in range(6)]
    ms = statistics.mean(tot)
    _, tf_burst, tf_sust, src = peaks()
    f_bwd_sparse = 2.5 * f_sparse
    f_lr_bwd = 2.0 * F.lowrank_flops(w.L, w.rank, w.head_dim, w.batch * w.heads)  # ~2x the forward's chain
    sparse_ms = st[2] + st[3]
    line = {"backward": w.name, "options": {k_: (v_ if not isinstance(v_, tuple) else "gated")
                                            for k_, v_ in var.items() if k_ != "gate" or v_ is not None},
            "ms_per_call": ms, "keep_blocks": keep_blocks,
            "stage_ms": dict(zip(("recompute_forward", "dout_copy_and_lists", "dq_kernel", "dkdv_kernel",
                                  "lowrank_grad", "-"), (round(x_, 4) for x_ in st))),
            "sparse_bwd": {"algorithmic_flops": f_bwd_sparse, "ms": sparse_ms,
                           "achieved_tflops": f_bwd_sparse / (sparse_ms * 1e-3) / 1e12,
                           "frac_of_burst": f_bwd_sparse / (sparse_ms * 1e-3) / 1e12 / tf_burst,
                           "peak": tf_burst, "peak_source": f"{src} burst bf16 (same rate as f16)"},
            "lowrank_bwd_flops": f_lr_bwd,
            "whole_call_tflops": (f_bwd_sparse + f_lr_bwd) / (ms * 1e-3) / 1e12,
            "train_step": {"ms": statistics.mean(t_fwd) + statistics.mean(t_bwd),
                           "forward_train_ms": statistics.mean(t_fwd),
                           "backward_saved_ms": statistics.mean(t_bwd),
                           "backward_saved_stage_ms": dict(zip(("-", "dout_copy_and_lists", "dq_kernel", "dkdv_kernel",
                                                                "lowrank_grad", "-"), (round(x_, 4) for x_ in sts)))},
            "clocks": clk}
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """The keep x rank sweep at the Wan2.1-1.3B shape on one GPU: per point, ms per call, effective
    TFLOP/s, the attention kernel's share of the call and its burst-peak roofline fraction, and the
    call's roofline fraction.  One JSON line per point (not the benchmark contract line)."""
    import torch
    from sparse_rank_hybrid_b200 import build as B
    from sparse_rank_hybrid_b200 import slra

    B.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
    for e in stage_ev:
        e.record()
    torch.cuda.synchronize()
    clocks = ClockSampler(0 if "CUDA_VISIBLE_DEVICES" not in os.environ else
                          int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[0]))
    clocks.start()
    for w in WL.sweep():
        _, _, prob, tensors = _problem(args, w, slra, dev, torch, stage_ev)
        ws = slra.alloc_workspace(prob, dev)
        out = torch.empty((w.batch, w.L, w.heads, w.head_dim), dtype=torch.float32, device=dev)
        q, k, v, A = tensors
        slra.attn_fwd(prob, q, k, v, A, out=out, workspace=ws)
        torch.cuda.synchronize()
        f_total, f_sparse, f_lr, f_sc, f_attn, keep_blocks = _work(w, prob, ws, slra, 3)
        step_ms, stage_ms = _timed_calls(slra, torch, prob, tensors, out, ws, stage_ev, args.steps, args.warmup,
                                         flush, stream)
        ms = statistics.mean(step_ms)
        stage_avg = [statistics.mean(x[i] for x in stage_ms) for i in range(6)]
        roof, call_roof = _rooflines(w, f_sparse, f_attn, stage_avg[5], ms)
        print(json.dumps({"sweep_point": w.name, "keep_frac": w.keep_frac, "keep_blocks": keep_blocks,
                          "rank": w.rank, "ms_per_call": ms, "tflops": f_total / (ms * 1e-3) / 1e12,
                          "attn_ms": stage_avg[5], "attn_share": stage_avg[5] / ms,
                          "attn_frac_burst": roof["frac"], "call_frac_burst": call_roof["frac"],
                          "prep_ms": round(sum(stage_avg[1:5]), 4)}), flush=True)
        del ws, out, tensors, q, k, v, A
    print(json.dumps({"sweep_clocks": clocks.stop()}), flush=True)


def load_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu capture, or None when there
    is none for this workload or the kernel source has changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f).get(workload)
        src = os.path.join(ROOT, "sparse_rank_hybrid_b200", "csrc", "attn_sm100.cu")
        with open(src, "rb") as f:
            current = hashlib.sha256(f.read()).hexdigest()
        return t["bytes"] if t and t.get("source_sha256") == current else None
    except (OSError, ValueError, KeyError, TypeError):
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--activation", default="relu", choices=sorted(ACTS), help="low-rank feature map")
    ap.add_argument("--lowrank-norope", action="store_true", help="low-rank branch without its RoPE")
    ap.add_argument("--linear-baseline", action="store_true",
                    help="full-width linear-attention branch: rank = head_dim, A = I, relu, no low-rank RoPE")
    ap.add_argument("--branches", default="both", choices=["both", "sparse", "lowrank"])
    ap.add_argument("--proj", default="shared", choices=list(PROJS),
                    help="query/key projection layout: one shared A, separate Pq/Pk, per head, or both")
    ap.add_argument("--fusion", default="sum", choices=["sum", "gated"],
                    help="combine the branches by their sum or by the token-wise gate (synthetic Wg, bg = -2)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (slra_attn_bwd) at the workload's shape (one JSON line)")
    ap.add_argument("--sweep", action="store_true",
                    help="time the 20 keep x rank points at the Wan2.1-1.3B shape (one JSON line each)")
    ap.add_argument("--rope-inside", action="store_true",
                    help="low-rank RoPE before the activation (the ordering RoLA's ablation compares against)")
    args = ap.parse_args()
    if args.rope_inside and (args.lowrank_norope or args.linear_baseline):
        ap.error("--rope-inside needs the low-rank RoPE")
    if args.fusion == "gated" and args.branches != "both":
        ap.error("--fusion gated needs both branches")
    if args.linear_baseline and args.proj != "shared":
        ap.error("--linear-baseline uses A = I (one shared projection)")
    w = WL.by_name(args.workload)
    if args.linear_baseline:
        args.lowrank_norope = True
        args.activation = "relu"
        w = w.with_(name=w.name + "-linear", rank=w.head_dim)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.backward:
        run_backward(args, w)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
