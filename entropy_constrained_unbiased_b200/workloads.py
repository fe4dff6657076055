"""Seeded synthetic inputs for the ECASQ solver.

This module draws input vectors only. It holds none of the solver's arithmetic
(no grid, no buckets, no DP), so that the oracle and the CUDA path can both be
fed from it without sharing any of the method.

The distributions are the synthetic families on which the ECASQ summary
evaluates (gist.science/pt/paper/2608.18147, §4 "Resultados Experimentais":
Normal, Lognormal, Student-t, sparse outliers). The five named workloads and
their sizes:

  small      1 x 1024      N(0,1)                        p=64   s=8   lambda=0.05
  weights    4096 x 4096   0.02 * Student-t(nu=4)        p=128  s=16  budget b=3.0
  gradients  256 x 2^20    N(0,1) * LogN(0,1) per row,   p=256  s=16  budget b=2.0
                           1% of entries x10
  sweep      1024 x 16384  Laplace(0,1)                  p=128  s=8   32 lambdas 10^(-4..0)
  mixture    64 x 65536    0.9 N(0,1) + 0.1 N(0,9)       p=512  s=32  lambda=0.01 (Hirschberg)
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    n: int
    d: int
    p: int
    s: int
    mode: str                      # "solve" | "budget" | "sweep"
    lam: float = 0.0               # fixed lambda ("solve")
    b: float = 0.0                 # entropy budget ("budget")
    steps: int = 30                # bisection steps ("budget")
    n_lambda: int = 1              # number of lambdas ("sweep")
    hirschberg: bool = False
    seed_encode: int = 1
    dist: str = "normal"

    def lambdas(self) -> np.ndarray:
        """[n, n_lambda] lambda table for "solve"/"sweep" workloads."""
        if self.mode == "sweep":
            k = np.arange(self.n_lambda, dtype=np.float64)
            lam = 10.0 ** (-4.0 + 4.0 * k / (self.n_lambda - 1))
            return np.broadcast_to(lam, (self.n, self.n_lambda)).copy()
        return np.full((self.n, 1), self.lam)


WORKLOADS = {
    "small": Workload("small", 0, 1, 1024, 64, 8, "solve", lam=0.05, dist="normal"),
    "weights": Workload("weights", 1, 4096, 4096, 128, 16, "budget", b=3.0, dist="student_t"),
    "gradients": Workload("gradients", 2, 256, 1 << 20, 256, 16, "budget", b=2.0, dist="grad"),
    "sweep": Workload("sweep", 3, 1024, 16384, 128, 8, "sweep", n_lambda=32, dist="laplace"),
    "mixture": Workload("mixture", 4, 64, 65536, 512, 32, "solve", lam=0.01, hirschberg=True,
                        dist="mixture"),
}
BY_INDEX = {w.index: w for w in WORKLOADS.values()}


def _row(dist: str, rng: np.random.Generator, d: int, scale: float) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(d, dtype=np.float32)
    if dist == "student_t":
        return (0.02 * rng.standard_t(4.0, size=d)).astype(np.float32)
    if dist == "laplace":
        return rng.laplace(0.0, 1.0, size=d).astype(np.float32)
    if dist == "mixture":
        wide = rng.random(d) < 0.1
        return (rng.standard_normal(d) * np.where(wide, 3.0, 1.0)).astype(np.float32)
    if dist == "lognormal":
        return rng.lognormal(0.0, 1.0, size=d).astype(np.float32)
    if dist in ("grad", "outlier"):
        z = rng.standard_normal(d, dtype=np.float32) * np.float32(scale)
        mask = rng.random(d, dtype=np.float32) < 0.01
        z[mask] *= np.float32(10.0)
        return z
    raise ValueError(dist)


def draw(dist: str, rng: np.random.Generator, n: int, d: int, rows: int | None = None) -> np.ndarray:
    """The first `rows` (default n) rows of an n x d float32 draw of one family.

    Rows are drawn one after another, so a prefix of rows does not depend on n
    beyond the per-row scales of the "grad" family, which are drawn first for all
    n rows.
    """
    rows = n if rows is None else min(rows, n)
    scale = rng.lognormal(0.0, 1.0, size=n) if dist == "grad" else np.ones(n)
    out = np.empty((rows, d), np.float32)
    for r in range(rows):
        out[r] = _row(dist, rng, d, float(scale[r]))
    return out


def make_inputs(w: Workload | str, rows: int | None = None, rank: int = 0) -> np.ndarray:
    """X for a named workload: [n, d] float32, or its first `rows` rows.

    Rank 0 draws the workload itself; rank r > 0 (multi-GPU weak scaling)
    draws its own vectors of the same family from the seed [index, r]."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    # The small workload is seeded with 0; the others with [index, 0].
    if rank == 0:
        rng = np.random.default_rng(0 if w.index == 0 else [w.index, 0])
    else:
        rng = np.random.default_rng([w.index, rank])
    return draw(w.dist, rng, w.n, w.d, rows)


def random_case(seed: int, n: int, d: int, dist: str = "normal") -> np.ndarray:
    """A seeded n x d test input of one family."""
    return draw(dist, np.random.default_rng([1000, seed]), n, d)


def pinned_range_rows(seed: int, n: int, d: int, lo: float, hi: float) -> np.ndarray:
    """n x d float32 rows, log-uniform between lo > 0 and hi with log-normal
    jitter, clipped to [lo, hi] and holding lo and hi themselves, so that every
    row covers exactly [lo, hi] (and has the same alphabet of the values
    representable in a given format over that range)."""
    rng = np.random.default_rng([2000, seed])
    X = np.exp(rng.uniform(np.log(lo), np.log(hi), size=(n, d)) + 0.3 * rng.standard_normal((n, d)))
    X = np.clip(X, lo, hi).astype(np.float32)
    X[:, 0], X[:, 1] = np.float32(lo), np.float32(hi)
    return X
