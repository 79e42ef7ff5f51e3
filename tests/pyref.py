"""Independent Python checkers used to pin the CPU oracle.

Nothing here is shared with the oracle or the CUDA library.  Each checker is a
different formulation of the same rule (a linear search of the whole key
array instead of a window probe, a textbook LRU list, exact rational
arithmetic instead of binary32 operations), so that a slip in the oracle's
indexing, ordering or rounding shows up as a disagreement.
"""
from __future__ import annotations

import collections
from fractions import Fraction

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def splitmix64(x: int) -> int:
    """SplitMix64 output for state x (Steele, Lea, Flood, OOPSLA 2014)."""
    z = (x + GAMMA) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def home(key: int, capacity: int) -> int:
    return splitmix64(key) % capacity


# ----------------------------------------------------------------------------
# Brute-force table: dict-free arrays, whole-array linear search for lookups.
# ----------------------------------------------------------------------------
class BruteTable:
    def __init__(self, capacity, dim, probes):
        self.C, self.D, self.P = capacity, dim, probes
        self.keys = [-1] * capacity
        self.last = [-1] * capacity
        self.M = np.zeros((capacity, dim), np.float32)

    def window(self, k):
        h = home(k, self.C)
        return [(h + j) % self.C for j in range(self.P)]

    def find(self, k):
        # linear search of the entire key array; a live key must sit in its window
        hits = [r for r in range(self.C) if self.keys[r] == k]
        assert len(hits) <= 1, "duplicate live key"
        if hits:
            assert hits[0] in self.window(k), "live key outside its probe window"
            return hits[0]
        return -1

    def lookup(self, ids):
        rows = np.array([self.find(int(k)) for k in ids], np.int32)
        return rows, (rows >= 0).astype(np.uint8)

    def writeback(self, ids, e, t):
        first = {}
        for i, k in enumerate(ids):
            first.setdefault(int(k), i)
        uniq = list(first)
        row = {}
        for k in uniq:
            r = self.find(k)
            if r >= 0:
                row[k] = r
                self.last[r] = t
        n_hit = len(row)
        missing = sorted(k for k in uniq if k not in row)
        n_evicted = 0
        for k in missing:
            cand = sorted(self.window(k), key=lambda r: (self.last[r], r))
            r = cand[0]
            if self.keys[r] != -1:
                n_evicted += 1
            self.keys[r] = k
            self.last[r] = t
            row[k] = r
        n_dropped = 0
        for k in uniq:
            r = row[k]
            if self.keys[r] != k:
                n_dropped += 1
                continue
            eh = self.M[r].copy()
            self.M[r] = eh - (eh - e[first[k]])  # numpy float32: one rounding per op
        return dict(n_ids=len(ids), n_unique=len(uniq), n_hit_unique=n_hit,
                    n_inserted=len(missing), n_evicted=n_evicted, n_dropped=n_dropped)


class TextbookLRU:
    """A capacity-bounded LRU cache kept as a recency-ordered list."""

    def __init__(self, capacity):
        self.cap = capacity
        self.od = collections.OrderedDict()

    def access(self, k):
        if k in self.od:
            self.od.move_to_end(k)
            return True, None
        victim = None
        if len(self.od) >= self.cap:
            victim, _ = self.od.popitem(last=False)
        self.od[k] = True
        return False, victim


class TextbookDirectMapped:
    """A direct-mapped cache: key k may only live in line index(k)."""

    def __init__(self, capacity, index):
        self.lines = [None] * capacity
        self.index = index

    def access(self, k):
        i = self.index(k)
        if self.lines[i] == k:
            return True
        self.lines[i] = k
        return False


# ----------------------------------------------------------------------------
# Exact binary32 rounding from rationals (for the quantiser pin).
# ----------------------------------------------------------------------------
def round_f32(x: Fraction) -> np.float32:
    """Round a rational to the nearest binary32, ties to even mantissa."""
    c = np.float32(float(x))
    best = None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        d = abs(Fraction(float(cand)) - x)
        if best is None or d < best[0] or (d == best[0] and (int(cand.view(np.uint32)) & 1) == 0):
            best = (d, cand)
    return np.float32(best[1])


def rne_int(x: Fraction) -> int:
    """Round a rational to the nearest integer, ties to even."""
    f = x.numerator // x.denominator
    rem = x - f
    if rem > Fraction(1, 2):
        return f + 1
    if rem < Fraction(1, 2):
        return f
    return f if f % 2 == 0 else f + 1


def quantize_exact(x: np.ndarray):
    """Per-row int8 with exactly-rounded binary32 steps, computed in rationals."""
    a = max(abs(Fraction(float(v))) for v in x)
    if a == 0:
        return np.zeros(x.size, np.int8), np.float32(0.0)
    scale = round_f32(a / 127)
    q = []
    for v in x:
        y = round_f32(Fraction(float(v)) / Fraction(float(scale)))
        r = rne_int(Fraction(float(y)))
        q.append(max(-127, min(127, r)))
    return np.array(q, np.int8), scale
