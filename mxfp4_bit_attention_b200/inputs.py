"""Seeded synthetic inputs shaped like video-DiT self-attention.

This module holds no arithmetic of the attention method: it only draws
random numbers and rounds them to the input dtype.  Both the CUDA path's
tests/bench and the CPU oracle's tests take their inputs from here.

Recipe (per workload; every draw comes from numpy PCG64 streams spawned from
``SeedSequence(seed)``: stream 0 draws the structure, stream 1 + t*BH + h
draws tensor t in (Q, K, V) for head h as an [N, d] fp32 standard normal
block):

* ``tiny``     B1 H1 N256 d64, fp32: Q, K, V ~ N(0, 1).
* ``outlier``  B1 H8 N4096 d128, bf16: Q, V ~ N(0, 1); K ~ N(0, 1) with four
               channels (``choice(d, 4)``, shared by all heads) scaled by 16
               plus a per-(head, token) offset mu ~ N(0, 0.5^2) on every channel.
* ``480p``     B1 H40 N32760 (21x30x52 latent tokens) d128, bf16: Q and K
               scaled per (head, channel) by exp(z), z ~ N(0, 1) (independent
               for Q and K); V ~ N(0, 1).
* ``720p``     B1 H40 N75600 (21x45x80) d128, bf16: as 480p plus 756 tokens
               (1%, ``choice(N, 756)``, shared by heads) whose Q and K rows are
               multiplied by 8.
* ``joint``    B1 H24 N119056 (33x45x80 video + 256 text) d128, bf16: per-channel
               scales exp(1.5 z); the last 256 tokens (text) have Q and K x4.

Structure draws happen first, in this order: per-channel scales for Q then K
([BH, d] each), then the channel/token index choices, then the offsets.
bf16 rounding is round-to-nearest-even of the fp32 draw.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str  # "bf16" or "fp32"
    seed: int
    key_tile: int = 64

    @property
    def BH(self) -> int:
        return self.B * self.H

    @property
    def flops(self) -> float:
        """4 * B * H * N^2 * d: the two N x N x d contractions of attention."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 256, 64, "fp32", 0),
    "outlier": Workload("outlier", 1, 8, 4096, 128, "bf16", 1),
    "480p": Workload("480p", 1, 40, 32760, 128, "bf16", 2),
    "720p": Workload("720p", 1, 40, 75600, 128, "bf16", 3),
    "joint": Workload("joint", 1, 24, 119056, 128, "bf16", 4),
}


def fp32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> 16) & np.uint32(1)
    return ((b + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_fp32(b: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _structure(w: Workload, rng: np.random.Generator):
    st = {}
    if w.name in ("480p", "720p"):
        st["sq"] = np.exp(rng.standard_normal((w.BH, w.d))).astype(np.float32)
        st["sk"] = np.exp(rng.standard_normal((w.BH, w.d))).astype(np.float32)
    if w.name == "joint":
        st["sq"] = np.exp(1.5 * rng.standard_normal((w.BH, w.d))).astype(np.float32)
        st["sk"] = np.exp(1.5 * rng.standard_normal((w.BH, w.d))).astype(np.float32)
    if w.name == "outlier":
        st["ch"] = rng.choice(w.d, 4, replace=False)
        st["mu"] = rng.normal(0.0, 0.5, (w.BH, w.N)).astype(np.float32)
    if w.name == "720p":
        st["hot"] = rng.choice(w.N, w.N // 100, replace=False)
    if w.name == "joint":
        st["text"] = np.arange(w.N - 256, w.N)
    return st


def _block(w: Workload, st: dict, t: int, h: int, seq: np.random.SeedSequence) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seq))
    z = rng.standard_normal((w.N, w.d), dtype=np.float32)
    if t == 0:  # Q
        if "sq" in st:
            z *= st["sq"][h]
        if "hot" in st:
            z[st["hot"]] *= np.float32(8.0)
        if "text" in st:
            z[st["text"]] *= np.float32(4.0)
    elif t == 1:  # K
        if "sk" in st:
            z *= st["sk"][h]
        if "ch" in st:
            z[:, st["ch"]] *= np.float32(16.0)
            z += st["mu"][h][:, None]
        if "hot" in st:
            z[st["hot"]] *= np.float32(8.0)
        if "text" in st:
            z[st["text"]] *= np.float32(4.0)
    return z


def generate(workload, heads=None, threads: int | None = None):
    """Draw Q, K, V for a workload.

    Returns a dict with ``q``, ``k``, ``v`` as arrays [BH', N, d]: uint16 bf16
    bit patterns for bf16 workloads, float32 for fp32 ones, where BH' covers
    ``heads`` (default: all heads).  Per-head draws are independent streams,
    so a subset of heads is identical to the same heads of the full draw.
    """
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    heads = list(range(w.BH)) if heads is None else list(heads)
    seqs = np.random.SeedSequence(w.seed).spawn(1 + 3 * w.BH)
    st = _structure(w, np.random.Generator(np.random.PCG64(seqs[0])))
    out_dtype = np.uint16 if w.dtype == "bf16" else np.float32
    res = {n: np.empty((len(heads), w.N, w.d), out_dtype) for n in ("q", "k", "v")}

    def job(args):
        t, i, h = args
        z = _block(w, st, t, h, seqs[1 + t * w.BH + h])
        res["qkv"[t]][i] = fp32_to_bf16_bits(z) if w.dtype == "bf16" else z

    jobs = [(t, i, h) for t in range(3) for i, h in enumerate(heads)]
    n = threads or min(16, os.cpu_count() or 1)
    with cf.ThreadPoolExecutor(n) as ex:
        list(ex.map(job, jobs))
    res["workload"] = w
    res["heads"] = heads
    return res


def as_fp32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Inputs as exact fp32 values (bf16 bits upcast)."""
    return bf16_bits_to_fp32(x) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def sample_rows(N: int, count: int = 64, seed: int = 12345, tile: int = 128) -> np.ndarray:
    """Query rows for sampled checks: the whole first tile's first rows, the
    ragged last tile, and random rows in between (sorted, unique)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    last0 = (N - 1) // tile * tile
    fixed = {0, 1, min(tile - 1, N - 1), last0, N - 1, max(N - 2, 0)}
    rest = rng.choice(N, max(count - len(fixed), 0), replace=False)
    return np.array(sorted(fixed | set(int(r) for r in rest)))[:max(count, len(fixed))]
