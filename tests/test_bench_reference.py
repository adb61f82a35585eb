"""The benchmark's reference arm (the fp64 oracle timed on the host cores) on the tiny workload: it
prints one JSON line with the contract's keys on rank 0 and nothing on other ranks (CPU only)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "0",
           "--workload", "tiny"] + extra
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [l for l in r.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("extra", [[], ["--proj", "separate-per-head"], ["--activation", "silu", "--lowrank-norope"],
                                   ["--fusion", "gated"], ["--rope-inside"]])
def test_reference_arm_line(extra):
    lines = _run(extra)
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["config"]["workload"] == "tiny"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_other_rank_is_silent():
    assert _run([], {"RANK": "1", "WORLD_SIZE": "2"}) == []
