"""Seeded synthetic inputs shared by the GPU path's tests/bench and the CPU oracle.

This module only draws random numbers and rounds them to bf16; it contains none of the attention
method's arithmetic.  The recipe stands in for real DiT activations (which are not available):
for each of q, k, v in that order, one N(0,1) centroid per (batch, head, frame, 4x4 spatial tile)
and per-token N(0,1) noise, X = 0.5*noise + centroid, rounded to bf16 (round-to-nearest-even).
The feature projection A ~ N(0, 1/head_dim) of shape [head_dim, rank] is drawn after v (or from its
own seed for the sweep workloads), also rounded to bf16.  Separate and/or per-head projections
(make_projections) come from a stream of their own, seeded with the workload seed + 5000, so the
q/k/v draws stay the same.

Arrays are returned as uint16 numpy arrays holding bf16 bit patterns, laid out [B, L, heads, D]
(token-major, as a DiT QKV projection emits them) and [D, rank] for A.
"""
from __future__ import annotations

import numpy as np

from .workloads import Workload


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest-even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _clustered(rng: np.random.Generator, B: int, heads: int, D: int, T: int, H: int, W: int) -> np.ndarray:
    th, tw = -(-H // 4), -(-W // 4)
    cent = rng.standard_normal((B, heads, T, th, tw, D), dtype=np.float32)
    noise = rng.standard_normal((B, T * H * W, heads, D), dtype=np.float32)
    # centroid of each token's tile, broadcast to [B, T, H, W, heads, D]
    c = np.repeat(np.repeat(cent, 4, axis=3), 4, axis=4)[:, :, :, :H, :W, :]
    c = c.transpose(0, 2, 3, 4, 1, 5)
    x = noise.reshape(B, T, H, W, heads, D)
    x *= np.float32(0.5)
    x += c
    return f32_to_bf16_bits(x.reshape(B, T * H * W, heads, D))


def make_inputs(w: Workload) -> dict[str, np.ndarray]:
    rng = np.random.Generator(np.random.PCG64(w.seed))
    out = {}
    for name in ("q", "k", "v"):
        out[name] = _clustered(rng, w.batch, w.heads, w.head_dim, w.T, w.H, w.W)
    arng = rng if w.a_seed is None else np.random.Generator(np.random.PCG64(w.a_seed))
    a = arng.standard_normal((w.head_dim, w.rank), dtype=np.float32) * np.float32(1.0 / np.sqrt(w.head_dim))
    out["A"] = f32_to_bf16_bits(a)
    return out


def make_custom(seed: int, B: int, L_or_grid, heads: int, D: int, R: int, scale: float = 1.0) -> dict[str, np.ndarray]:
    """Plain Gaussian inputs (no clustering) for edge-case shapes; grid = (T, H, W)."""
    T, H, W = L_or_grid
    rng = np.random.Generator(np.random.PCG64(seed))
    L = T * H * W
    out = {n: f32_to_bf16_bits(rng.standard_normal((B, L, heads, D), dtype=np.float32) * np.float32(scale))
           for n in ("q", "k", "v")}
    out["A"] = f32_to_bf16_bits(rng.standard_normal((D, R), dtype=np.float32) * np.float32(1.0 / np.sqrt(D)))
    return out


def make_projections(seed: int, heads: int, D: int, R: int, separate: bool, per_head: bool) -> np.ndarray:
    """Projection argument for separate (Pq, Pk) and/or per-head projections: bf16 bits of shape
    [1 + separate, heads if per_head else 1, D, R], query projections first, each entry ~ N(0, 1/D)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (2 if separate else 1, heads if per_head else 1, D, R)
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(1.0 / np.sqrt(D)))


def make_dout(seed: int, B: int, L: int, heads: int, D: int, scale: float = 1.0) -> np.ndarray:
    """A seeded upstream gradient dout ~ N(0, scale^2), fp32 [B, L, heads, D], for the backward pass."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((B, L, heads, D), dtype=np.float32) * np.float32(scale)
