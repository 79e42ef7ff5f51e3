"""Seeded synthetic inputs for the Memory Layer workloads.

This module only *draws* data: item-ID streams, item-tower targets ``e`` and the
always-on (author) feature table and author ids.  It holds none of the table
arithmetic (no start-slot hash, probing, dedup, eviction, Writeback or
quantisation); both the CUDA path and the CPU oracle receive its arrays as
plain inputs.

Stand-ins (the pages' traffic is Instagram Reels production data, which is not
public):

* Item popularity is power-law skewed ("Memory Layer: Train the In-Model Cache
  for Recommendation Models", section 3 reports a 99.5% cache hit rate on such
  traffic; "MP-Rec", caching section, and "DLRMv4 training benchmark", dataset
  section, both describe power-law / skewed ID access), so ranks are drawn from
  a truncated Zipf law P(r) ~ r^-alpha, r = 1..N, by Hoermann-Derflinger
  rejection-inversion (W. Hoermann and G. Derflinger, "Rejection-inversion to
  generate variates from monotone discrete distributions", ACM TOMACS 6(3),
  1996).  Rank r maps to item key r-1.
* "Fresh" never-seen items (new uploads, the cold-start case the Memory Layer
  page motivates in section 1) get keys N + c with a global counter c.
* Item-tower targets are e ~ N(0, 1) fp32, 512-d as on the Memory Layer page
  (section 2) and the DLRMv4 page (512-d fp32 tables).

Draws use numpy's PCG64 seeded with small integer tuples, so every array is
reproducible from (workload, stream, step).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Number of distinct item-tower target batches per workload; step t uses batch
# t mod E_POOL.  The values of e never change which rows are touched, so the
# pool only bounds input-generation time and memory for long runs.
E_POOL = 8

_U64 = np.uint64
_MASK64 = (1 << 64) - 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload (table shape + per-step ID stream recipe)."""

    name: str
    cfg_id: int
    capacity: int
    dim: int
    probes: int
    steps: int
    # ids per step that go through lookup + gather (a prefix of the merged batch)
    labeled: int
    # extra unlabeled candidate-pool ids appended after the labeled ones (multi-table)
    pool: int
    zipf_alpha: float
    zipf_keys: int
    fresh_frac: float = 0.0
    # always-on (author) table: rows x dim, None = no concat
    ao_rows: int = 0
    ao_dim: int = 0
    ao_kind: Optional[str] = None  # "mod" (key mod ao_rows) or "mix" (splitmix64(key) mod ao_rows)
    ao_std: float = 0.1

    @property
    def batch(self) -> int:
        return self.labeled + self.pool

    @property
    def n_fresh(self) -> int:
        # fresh never-seen keys per step (part of the labeled stream when pool == 0)
        return int(round(self.fresh_frac * self.labeled)) if self.pool == 0 else 0

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Sizes follow the configurations the hot path is quoted on.
CFG1_TINY = Workload("tiny_c4096_d64_p4", 1, capacity=4096, dim=64, probes=4, steps=8,
                     labeled=256, pool=0, zipf_alpha=1.05, zipf_keys=10_000,
                     ao_rows=512, ao_dim=16, ao_kind="mod")
CFG2_1M = Workload("c1m_d512_p8_zipf1.1_fresh15", 2, capacity=1 << 20, dim=512, probes=8,
                   steps=100, labeled=65_536, pool=0, zipf_alpha=1.1, zipf_keys=20_000_000,
                   fresh_frac=0.15)
CFG3_MULTI = Workload("multitable_c1m_d512_p8_lab32768_pool131072_zipf0.9_author128", 3,
                      capacity=1 << 20, dim=512, probes=8, steps=100, labeled=32_768,
                      pool=131_072, zipf_alpha=0.9, zipf_keys=5_000_000,
                      ao_rows=1 << 20, ao_dim=128, ao_kind="mix")
CFG4_16M = Workload("c16m_d512_p8_zipf1.2_fresh20", 4, capacity=1 << 24, dim=512, probes=8,
                    steps=200, labeled=262_144, pool=0, zipf_alpha=1.2,
                    zipf_keys=200_000_000, fresh_frac=0.2)
# Serving/export (after the multi-table state): rows written in the last 50 steps
# are exported; then 4096 requests x 1024 candidates are served from the snapshot.
CFG5_SERVE_SINCE = 50
CFG5_REQUESTS = 4096
CFG5_CANDIDATES = 1024
CFG5_ALPHA = 0.9
CFG5_KEYS = 5_000_000

WORKLOADS = {1: CFG1_TINY, 2: CFG2_1M, 3: CFG3_MULTI, 4: CFG4_16M}


def _rng(*entropy: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(list(entropy)))


# --------------------------------------------------------------------------
# Zipf(alpha) over ranks 1..N by rejection-inversion.
#
# The unnormalised mass of rank k is f(k) = k^-alpha.  F(x) = int_1^x t^-alpha dt
# is the integral of the continuous envelope f(x); because f is convex and
# decreasing, the envelope mass on [k - 1/2, k + 1/2] is at least f(k).  A
# uniform u on [F(3/2) - f(1), F(N + 1/2)] is inverted to x = F^-1(u) and
# rounded to k; k is accepted when u lies in the top f(k) of its cell, i.e.
# u >= F(k + 1/2) - f(k).  Each k is thus accepted with probability mass
# exactly f(k) (rank 1's cell is cut to length f(1) so it is always accepted).
# --------------------------------------------------------------------------
def _zipf_F(x: np.ndarray, a: float) -> np.ndarray:
    lx = np.log(x)
    if a == 1.0:
        return lx
    return np.expm1((1.0 - a) * lx) / (1.0 - a)


def _zipf_Finv(u: np.ndarray, a: float) -> np.ndarray:
    if a == 1.0:
        return np.exp(u)
    return np.exp(np.log1p((1.0 - a) * u) / (1.0 - a))


def zipf_ranks(rng: np.random.Generator, alpha: float, n_keys: int, size: int) -> np.ndarray:
    """``size`` iid ranks in [1, n_keys] with P(r) proportional to r^-alpha."""
    a = float(alpha)
    lo = float(_zipf_F(np.array([1.5]), a)[0]) - 1.0
    hi = float(_zipf_F(np.array([n_keys + 0.5]), a)[0])
    out = np.empty(size, dtype=np.int64)
    filled = 0
    while filled < size:
        need = size - filled
        m = int(need * 1.15) + 64
        u = lo + rng.random(m) * (hi - lo)
        x = _zipf_Finv(u, a)
        k = np.clip(np.floor(x + 0.5), 1, n_keys)
        accept = u >= _zipf_F(k + 0.5, a) - np.power(k, -a)
        k = k[accept].astype(np.int64)[:need]
        out[filled:filled + k.size] = k
        filled += k.size
    return out


def zipf_keys(rng: np.random.Generator, alpha: float, n_keys: int, size: int) -> np.ndarray:
    return zipf_ranks(rng, alpha, n_keys, size) - 1


def splitmix64_np(x: np.ndarray) -> np.ndarray:
    """SplitMix64 generator output for state ``x`` (G. Steele, D. Lea, C. Flood,
    "Fast splittable pseudorandom number generators", OOPSLA 2014).  Used here
    only as the data scrambler that assigns synthetic author ids to items."""
    with np.errstate(over="ignore"):
        z = x.astype(_U64) + _U64(0x9E3779B97F4A7C15)
        z = (z ^ (z >> _U64(30))) * _U64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> _U64(27))) * _U64(0x94D049BB133111EB)
        return z ^ (z >> _U64(31))


# --------------------------------------------------------------------------
# Per-step inputs
# --------------------------------------------------------------------------
def step_ids(w: Workload, t: int) -> np.ndarray:
    """int64 item ids of step t (labeled ids first, then the candidate pool)."""
    if w.pool:
        lab = zipf_keys(_rng(w.cfg_id, 1, t), w.zipf_alpha, w.zipf_keys, w.labeled)
        pool = zipf_keys(_rng(w.cfg_id, 2, t), w.zipf_alpha, w.zipf_keys, w.pool)
        return np.ascontiguousarray(np.concatenate([lab, pool]))
    rng = _rng(w.cfg_id, 1, t)
    nf = w.n_fresh
    z = zipf_keys(rng, w.zipf_alpha, w.zipf_keys, w.labeled - nf)
    if nf:
        fresh = np.int64(w.zipf_keys) + np.int64(t) * nf + np.arange(nf, dtype=np.int64)
        ids = np.concatenate([z, fresh])
        ids = ids[rng.permutation(ids.size)]
    else:
        ids = z
    return np.ascontiguousarray(ids.astype(np.int64))


def step_e(w: Workload, t: int, rows: Optional[int] = None) -> np.ndarray:
    """fp32 item-tower targets e[B][D] of step t, e ~ N(0, 1)."""
    b = w.batch if rows is None else rows
    return _rng(w.cfg_id, 9, t % E_POOL).standard_normal((b, w.dim), dtype=np.float32)


def author_table(w: Workload) -> Optional[np.ndarray]:
    """Always-on author embedding table [ao_rows][ao_dim] fp32 ~ N(0, ao_std)."""
    if not w.ao_kind:
        return None
    t = _rng(w.cfg_id, 7).standard_normal((w.ao_rows, w.ao_dim), dtype=np.float32)
    return (t * np.float32(w.ao_std)).astype(np.float32)


def author_rows(w: Workload, ids: np.ndarray) -> Optional[np.ndarray]:
    """Synthetic author id of each item (row of the always-on table), int32."""
    if not w.ao_kind:
        return None
    if w.ao_kind == "mod":
        return (ids % w.ao_rows).astype(np.int32)
    return (splitmix64_np(ids) % _U64(w.ao_rows)).astype(np.int32)


def serve_candidates(n_requests: int = CFG5_REQUESTS, n_cand: int = CFG5_CANDIDATES,
                     alpha: float = CFG5_ALPHA, n_keys: int = CFG5_KEYS, seed: int = 5000) -> np.ndarray:
    """Serving candidates: n_requests x n_cand item ids, Zipf(alpha) over n_keys."""
    return zipf_keys(_rng(5, seed), alpha, n_keys, n_requests * n_cand)


def math_zipf_pmf(alpha: float, n_keys: int) -> np.ndarray:
    """Exact truncated Zipf pmf over ranks 1..n_keys (for generator self-checks)."""
    r = np.arange(1, n_keys + 1, dtype=np.float64)
    p = r ** (-alpha)
    return p / math.fsum(p)
