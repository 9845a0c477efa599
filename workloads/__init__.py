"""Seeded synthetic inputs for the exact-budget soft top-k workloads.

This module only draws numbers: it holds none of the method's arithmetic, so
both the CUDA path's tests/benchmark and the fp64 oracle can consume the very
same bytes without sharing any code of the method.

Workloads (the score distributions, budgets and temperatures of the method's
headline measurements; "Fast LapSum: Exact Differentiable Top-k at Million
Scale", abstract and technical summary section 4.1, where solver times are
quoted at 1e6, 1e7 and 1e8 scores; the 1024x1024 'pixel' case stands in for
the megapixel sparse-attack workload of section 4.2, whose images and
classifier are not available here):

  n4096         1 x 4096        N(0,1)                            k=64      t=0.05
  rows1024      1024 x 32768    N(0,1) per row                    k=256     t=0.1
  pixels1m      1 x 1,048,576   99% N(0,0.1^2); 10486 random      k=210     t=0.01
                                positions N(2,0.5^2)
  laplace1e7    1 x 1e7         Laplace(0,1)                      k=1e5     t=0.05
  levels1e8     1 x 1e8         256 levels of U(-4,4), level i ->  k=1e6     t=0.1
                                -4+(i+1/2)/32, sorted descending
  levels1e8_shuffled            the same scores in random order     k=1e6     t=0.1

Every workload draws its scores, its random positions and its upstream
gradient g ~ N(0,1) from three independent PCG64 streams spawned from one
SeedSequence(seed).
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = ["Workload", "WORKLOADS", "scores", "upstream_grad", "small_case", "streams"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    rows: int
    n: int
    k: float
    t: float
    dist: str          # "normal" | "pixel_mix" | "laplace" | "levels256_desc"
    path: str          # the solver path the workload exercises
    note: str = ""

    @property
    def units(self) -> int:
        """Scores processed by one forward (or forward+VJP) call."""
        return self.rows * self.n


WORKLOADS: dict[str, Workload] = {
    w.name: w for w in [
        Workload("n4096", 1, 4096, 64.0, 0.05, "normal", "full-sort (one CTA)"),
        Workload("rows1024", 1024, 32768, 256.0, 0.1, "normal",
                 "per-row segmented full sort"),
        Workload("pixels1m", 1, 1_048_576, 210.0, 0.01, "pixel_mix",
                 "bracketing + certification"),
        Workload("laplace1e7", 1, 10_000_000, 100_000.0, 0.05, "laplace",
                 "bracketing + band select + certification"),
        Workload("levels1e8", 1, 100_000_000, 1_000_000.0, 0.1, "levels256_desc",
                 "bracketing (+ forced full-sort fallback run)"),
        Workload("batch64x1m", 64, 1_048_576, 10_486.0, 0.05, "normal",
                 "batched bracketing (64 rows of 2^20, k = 1% of each row)"),
        Workload("levels1e8_shuffled", 1, 100_000_000, 1_000_000.0, 0.1, "levels256_shuffled",
                 "the levels1e8 scores in random order (every chunk of the row mixes levels)"),
    ]
}


def streams(seed: int = 0) -> tuple[np.random.Generator, np.random.Generator, np.random.Generator]:
    """(scores, positions, grad) generators: independent PCG64 streams."""
    ss = np.random.SeedSequence(seed).spawn(3)
    return tuple(np.random.Generator(np.random.PCG64(s)) for s in ss)  # type: ignore[return-value]


def _levels256_desc(rng: np.random.Generator, n: int) -> np.ndarray:
    # A float32 draw u in [0,1) has 24-bit granularity, so floor(256*u) hits each
    # of the 256 levels with probability exactly 1/256.  The array is stored
    # sorted descending, so only the level counts matter: draw them directly.
    counts = rng.multinomial(n, np.full(256, 1.0 / 256.0))
    values = (-4.0 + (np.arange(256, dtype=np.float64) + 0.5) / 32.0).astype(np.float32)
    return np.repeat(values[::-1], counts[::-1])


def _draw(dist: str, rows: int, n: int, rs: np.random.Generator, rp: np.random.Generator) -> np.ndarray:
    if dist == "normal":
        return rs.standard_normal((rows, n), dtype=np.float32)
    if dist == "laplace":
        return rs.laplace(0.0, 1.0, (rows, n)).astype(np.float32)
    if dist == "pixel_mix":
        out = np.empty((rows, n), dtype=np.float32)
        m = int(round(0.01 * n))
        for i in range(rows):
            row = (0.1 * rs.standard_normal(n, dtype=np.float32)).astype(np.float32)
            pos = rp.choice(n, size=m, replace=False)
            row[pos] = (2.0 + 0.5 * rs.standard_normal(m, dtype=np.float32)).astype(np.float32)
            out[i] = row
        return out
    if dist == "levels256_desc":
        return np.stack([_levels256_desc(rs, n) for _ in range(rows)])
    if dist == "levels256_shuffled":   # the same multiset of levels, then a random permutation
        out = np.stack([_levels256_desc(rs, n) for _ in range(rows)])
        for i in range(rows):
            rp.shuffle(out[i])
        return out
    if dist == "uniform":
        return rs.uniform(-1.0, 1.0, (rows, n)).astype(np.float32)
    raise ValueError(f"unknown distribution {dist!r}")


def scores(w: Workload | str, seed: int = 0) -> np.ndarray:
    """float32 [rows, n] scores of a workload, C-contiguous."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    rs, rp, _ = streams(seed)
    return np.ascontiguousarray(_draw(w.dist, w.rows, w.n, rs, rp))


def upstream_grad(w: Workload | str, seed: int = 0) -> np.ndarray:
    """float32 [rows, n] upstream gradient g ~ N(0,1)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    _, _, rg = streams(seed)
    return rg.standard_normal((w.rows, w.n), dtype=np.float32)


def small_case(dist: str, rows: int, n: int, seed: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """Scores and upstream grad of one of the workload distributions at a reduced size."""
    w = Workload(f"{dist}-{rows}x{n}", rows, n, 1.0, 1.0, dist, "")
    return scores(w, seed), upstream_grad(w, seed)
