"""Seeded synthetic inputs for top-p routed block-sparse attention.

This module holds no arithmetic of the method: it only draws inputs (and
names the workload shapes).  Both the oracle side and the CUDA side consume
exactly the bytes it returns.

Inputs are drawn with numpy's PCG64 (``default_rng(seed)``) in fp32 and rounded
to bf16 with round-to-nearest-even; arrays are returned as uint16 bit patterns
of shape [B, H, N, d].

Two distributions:
  * ``iid``: Q, K, V ~ N(0, 1).
  * ``structured`` (video-latent-like): token t <-> (tau, y, x) on a T x Y x X
    grid, row-major with tau slowest.  Per head h, 8 low-frequency sinusoids
    j with integer frequencies (k_tau, k_y, k_x) uniform in {-2..2}^3 \\ {0},
    phase ~ U(0, 2pi) and direction u_j ~ N(0, I/8) give
      f_h(t) = sum_j u_j sin(2 pi (k_tau tau/T + k_y y/Y + k_x x/X) + phase_j).
    Q = N(0,1) + s_h f_h and K = N(0,1) + s_h f_h (the same f_h), V ~ N(0,1),
    with s_h drawn per head, so routing concentration varies across heads.
The pages' own workloads (Wan2.2 I2V, HunyuanVideo latents) are not available;
these shapes stand in for them.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    bs: int
    p: float
    causal: bool = False
    dist: str = "iid"                 # "iid" or "structured"
    grid: tuple | None = None         # (T, Y, X) for structured inputs
    head_scale: tuple | None = None   # ("uniform", lo, hi) or ("const", v)
    seed: int = 0

    @property
    def nb(self) -> int:
        return -(-self.N // self.bs)

    @property
    def rows(self) -> int:
        return self.B * self.H * self.nb

    def describe(self) -> dict:
        d = dataclasses.asdict(self)
        d["nb"] = self.nb
        return d


TINY = Workload("tiny", B=1, H=2, N=512, d=64, bs=64, p=0.9, seed=0)
VIDEO = Workload("video_dit", B=1, H=40, N=21 * 30 * 52, d=128, bs=128, p=0.9, dist="structured",
                 grid=(21, 30, 52), head_scale=("uniform", 0.5, 4.0), seed=1)
DENSE = Workload("dense", B=2, H=16, N=16384, d=128, bs=128, p=1.0, seed=2)
DENSE_CAUSAL = dataclasses.replace(DENSE, name="dense_causal", causal=True)
LONG = Workload("long_video", B=1, H=24, N=33 * 45 * 80, d=128, bs=128, p=0.8, dist="structured",
                grid=(33, 45, 80), head_scale=("uniform", 0.5, 4.0), seed=3)

# Block 64 on the video shape (a measurement case beside the named configs: the
# pages' video workload, routed and attended in blocks of 64 tokens).
VIDEO_BS64 = dataclasses.replace(VIDEO, name="video_dit_bs64", bs=64)


def sweep() -> list[Workload]:
    """B1 H8 N32768 on a 16x32x64 grid; d x p x head-scale spread (20 runs)."""
    out = []
    idx = 0
    for d in (64, 128):
        for spread in (("const", 1.0), ("uniform", 0.5, 8.0)):
            for p in (0.5, 0.7, 0.9, 0.95, 1.0):
                tag = "s1" if spread[0] == "const" else "s05_8"
                out.append(Workload(f"sweep_d{d}_{tag}_p{p}", B=1, H=8, N=32768, d=d, bs=128, p=p,
                                    dist="structured", grid=(16, 32, 64), head_scale=spread, seed=100 + idx))
                idx += 1
    return out


ALL = {w.name: w for w in [TINY, VIDEO, DENSE, DENSE_CAUSAL, LONG, VIDEO_BS64] + sweep()}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bit patterns."""
    u = np.array(x, dtype=np.float32, copy=True, order="C").view(np.uint32)
    t = u >> np.uint32(16)
    t &= np.uint32(1)
    t += np.uint32(0x7FFF)
    u += t
    del t
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def _structure(rng: np.random.Generator, w: Workload) -> np.ndarray:
    """Per-head smooth field s_h * f_h(t): fp32 [H, N, d] (shared by every batch entry)."""
    T, Y, X = w.grid
    if T * Y * X != w.N:
        raise ValueError(f"grid {w.grid} does not have {w.N} tokens")
    kind = w.head_scale[0]
    if kind == "uniform":
        s = rng.uniform(w.head_scale[1], w.head_scale[2], size=w.H)
    else:
        s = np.full(w.H, float(w.head_scale[1]))
    t = np.arange(w.N)
    tau = (t // (Y * X)).astype(np.float64)
    y = ((t // X) % Y).astype(np.float64)
    x = (t % X).astype(np.float64)
    field = np.empty((w.H, w.N, w.d), dtype=np.float32)
    for h in range(w.H):
        freqs = []
        while len(freqs) < 8:
            f = rng.integers(-2, 3, size=3)
            if np.any(f != 0):
                freqs.append(f)
        freqs = np.asarray(freqs, dtype=np.float64)
        phase = rng.uniform(0.0, 2.0 * math.pi, size=8)
        u = rng.standard_normal(size=(8, w.d)) / math.sqrt(8.0)
        arg = 2.0 * math.pi * (np.outer(tau, freqs[:, 0]) / T + np.outer(y, freqs[:, 1]) / Y
                               + np.outer(x, freqs[:, 2]) / X) + phase[None, :]
        field[h] = (s[h] * (np.sin(arg) @ u)).astype(np.float32)
    return field


def generate(w: Workload, seed: int | None = None):
    """Q, K, V as bf16 bit patterns, each uint16 [B, H, N, d]."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.N, w.d)
    if w.dist == "structured":
        field = _structure(rng, w)
        q = rng.standard_normal(size=shape, dtype=np.float32)
        q += field[None]
        Q = f32_to_bf16_bits(q)
        del q
        k = rng.standard_normal(size=shape, dtype=np.float32)
        k += field[None]
        K = f32_to_bf16_bits(k)
        del k
        V = _normal_bf16(rng, shape)
    elif w.dist == "iid":
        Q = _normal_bf16(rng, shape)
        K = _normal_bf16(rng, shape)
        V = _normal_bf16(rng, shape)
    else:
        raise ValueError(w.dist)
    return Q, K, V


def sample_tokens(w: Workload, per_head_blocks: int = 2, seed: int = 12345, all_heads: bool = True,
                  rows_per_block: int | None = None) -> np.ndarray:
    """Flat token indices (b*H+h)*N + t covering query block 0, the last (ragged)
    query block and ``per_head_blocks`` seeded random query blocks of every head."""
    rng = np.random.default_rng(seed)
    toks = []
    for bh in range(w.B * w.H):
        blocks = {0, w.nb - 1}
        if w.nb > 2:
            blocks.update(int(b) for b in rng.choice(np.arange(1, w.nb - 1), size=min(per_head_blocks, w.nb - 2),
                                                     replace=False))
        for qb in sorted(blocks):
            t0, t1 = qb * w.bs, min(w.N, (qb + 1) * w.bs)
            ts = np.arange(t0, t1)
            if rows_per_block is not None and ts.size > rows_per_block:
                ts = np.sort(rng.choice(ts, size=rows_per_block, replace=False))
            toks.append(bh * w.N + ts)
    return np.concatenate(toks).astype(np.int64)
