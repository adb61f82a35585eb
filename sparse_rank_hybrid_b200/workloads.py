"""Named synthetic workloads for the 3D-RoPE sparse + low-rank hybrid attention forward.

Each workload is a video-DiT attention shape from the RoLA / RoPeSLR pages: a latent grid T x H x W
flattened to L = T*H*W tokens (RoLA, "3 Preliminary", full attention), `heads` attention heads of
width `head_dim`, a low-rank width `rank`, a block size and a kept fraction of key blocks
(90% sparsity = keep 10%, RoLA abstract).  The seeds fix the synthetic clustered-Gaussian inputs that
stand in for the real Wan2.1 / HunyuanVideo activations (see `inputs.py`).
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    T: int
    H: int
    W: int
    rank: int
    block: int
    keep_frac: float
    seed: int
    a_seed: int | None = None  # None: A is drawn from the q/k/v stream after v

    @property
    def L(self) -> int:
        return self.T * self.H * self.W

    @property
    def nb(self) -> int:
        return -(-self.L // self.block)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# Tiny case: 4x8x8 grid, 2 heads of width 64, rank 16, block 64, keep 2 of 4 key blocks.
TINY = Workload("tiny", 1, 2, 64, 4, 8, 8, 16, 64, 0.5, 1001)
# Wan2.1-1.3B at 480p: latent 21x30x52, 12 heads of width 128.
WAN_1_3B = Workload("wan2.1-1.3b-480p", 1, 12, 128, 21, 30, 52, 32, 128, 0.10, 1002)
# Wan2.1-14B at 720p / 81 frames: latent 21x45x80 = 75,600 tokens, 40 heads.
WAN_14B = Workload("wan2.1-14b-720p", 1, 40, 128, 21, 45, 80, 32, 128, 0.10, 1003)
# HunyuanVideo-13B long sequence: latent 33x45x80 = 118,800 tokens, 24 heads, rank 64.
HUNYUAN = Workload("hunyuanvideo-13b-long", 1, 24, 128, 33, 45, 80, 64, 128, 0.10, 1004)

MAIN = {w.name: w for w in (TINY, WAN_1_3B, WAN_14B, HUNYUAN)}


def sweep() -> list[Workload]:
    """Sparsity x rank sweep at the Wan2.1-1.3B shape: q/k/v from seed 1002, A from seed 1002 + r."""
    out = []
    for keep in (0.05, 0.10, 0.20, 0.50, 1.00):
        for r in (16, 32, 64, 128):
            out.append(WAN_1_3B.with_(name=f"sweep-keep{int(round(keep * 100))}-r{r}",
                                      keep_frac=keep, rank=r, a_seed=1002 + r))
    return out


def by_name(name: str) -> Workload:
    if name in MAIN:
        return MAIN[name]
    for w in sweep():
        if w.name == name:
            return w
    raise KeyError(name)
