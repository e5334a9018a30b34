"""Seeded synthetic inputs for the Fast LapSum soft top-k workloads.

This module holds only input generation: it draws scores ``r`` and upstream
gradients ``v`` and describes the workload shapes.  It contains none of the
operator's arithmetic, so both the CPU oracle's tests and the CUDA path's
tests and benchmark can use it without sharing any of the method.

Recipe (one ``numpy.random.default_rng(seed)`` PCG64 stream per workload):
draw all of ``r`` first, then all of ``v``, both in chunks of ``CHUNK``
elements over the row-major ``B x n`` array; each value is drawn in fp64 and
cast to fp32.  Within a chunk of ``r`` the draws are, per distribution:

* ``normal``       standard_normal(c)
* ``normal_q64``   round(standard_normal(c) * 64) / 64 (round half to even);
                   the result is exact in fp32 and has many exact ties
* ``abs_t3``       |standard_t(3, c)| (heavy right tail)
* ``mix_nu``       sel = random(c) < 0.5, a = standard_normal(c),
                   u = uniform(-4, 4, c); r = where(sel, a, u)

``v`` is standard_normal everywhere.  The distributions stand in for the data
the pages' applications use (MoE router logits, memory-selection scores, the
per-pixel mask of a 3x1024x1088 image, and a synthetic 10^8-score vector); no
dataset is read.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

CHUNK = 1 << 22


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    n: int
    k: float
    t: float
    dist: str
    path: str  # solver family the workload exercises: "onchip" (n <= 4096), "radix", "bracket"
    desc: str

    @property
    def elements(self) -> int:
        return self.B * self.n


WORKLOADS = {
    "single_row_n1024": Workload(
        "single_row_n1024", 1, 1024, 10.0, 0.1, "normal", "onchip",
        "single row n=1024, k=10, t=0.1, r ~ N(0,1)"),
    "moe_router_16384x256": Workload(
        "moe_router_16384x256", 16384, 256, 8.0, 0.05, "normal", "onchip",
        "MoE-routing batch 16384 rows x 256, k=8, t=0.05, r ~ N(0,1)"),
    "memory_select_256x65536": Workload(
        "memory_select_256x65536", 256, 65536, 1024.0, 0.02, "normal_q64", "radix",
        "memory-selection batch 256 rows x 65536, k=1024, t=0.02, r = N(0,1) quantised to 1/64"),
    "adv_mask_3342336": Workload(
        "adv_mask_3342336", 1, 3 * 1024 * 1088, 600.0, 0.01, "abs_t3", "bracket",
        "adversarial-mask row n=3*1024*1088, k=600, t=0.01, r = |Student-t(3)|"),
    "extreme_1e8": Workload(
        "extreme_1e8", 1, 100_000_000, 100_000.0, 0.005, "mix_nu", "bracket",
        "extreme-scale row n=1e8, k=1e5, t=0.005, r ~ 50/50 N(0,1) / U(-4,4)"),
}

# The five workloads in the order the benchmark table lists them.
ORDER = ["single_row_n1024", "moe_router_16384x256", "memory_select_256x65536",
         "adv_mask_3342336", "extreme_1e8"]


def _draw_scores(rng: np.random.Generator, dist: str, c: int) -> np.ndarray:
    if dist == "normal":
        x = rng.standard_normal(c)
    elif dist == "normal_q64":
        x = np.round(rng.standard_normal(c) * 64.0) / 64.0
    elif dist == "abs_t3":
        x = np.abs(rng.standard_t(3, c))
    elif dist == "mix_nu":
        sel = rng.random(c) < 0.5
        a = rng.standard_normal(c)
        u = rng.uniform(-4.0, 4.0, c)
        x = np.where(sel, a, u)
    else:
        raise ValueError(f"unknown score distribution {dist!r}")
    return x.astype(np.float32)


def make_inputs(w: Workload | str, seed: int = 0, with_v: bool = True):
    """Return (r, v) as float32 arrays of shape (B, n); v is None if not asked for."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    total = w.B * w.n
    rng = np.random.default_rng(seed)
    r = np.empty(total, dtype=np.float32)
    for s in range(0, total, CHUNK):
        c = min(CHUNK, total - s)
        r[s:s + c] = _draw_scores(rng, w.dist, c)
    v = None
    if with_v:
        v = np.empty(total, dtype=np.float32)
        for s in range(0, total, CHUNK):
            c = min(CHUNK, total - s)
            v[s:s + c] = rng.standard_normal(c).astype(np.float32)
        v = v.reshape(w.B, w.n)
    return r.reshape(w.B, w.n), v


def random_rows(seed: int, B: int, n: int, dist: str = "normal", scale: float = 1.0):
    """Small seeded (r, v) pairs for unit and parity tests."""
    rng = np.random.default_rng(seed)
    r = np.empty((B, n), dtype=np.float32)
    for i in range(B):
        r[i] = _draw_scores(rng, dist, n) * np.float32(scale)
    v = rng.standard_normal((B, n)).astype(np.float32)
    return r, v


def input_digest(a: np.ndarray) -> str:
    """Short content hash, stored beside expected values to catch generator drift."""
    import hashlib
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()[:16]
