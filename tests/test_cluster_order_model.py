"""The insert order the GPU's cluster placement relies on, checked on the CPU.

Missing ids must be inserted as if one at a time in ascending key order (the
victim being the smallest (last-write step, row) of the id's window).  The GPU
path instead cuts the ring of occupied start slots wherever two consecutive
ones are P or more apart, and places each resulting cluster's ids in ascending
order, clusters independently.  This test restates that cluster rule in
plain Python and checks, on thousands of random small tables (wrapped
windows, heavy eviction, ids evicted again in their own step, rings the
windows cover entirely), that it leaves exactly the identity map and
last-write steps of the oracle's sequential insert.
"""
import numpy as np
import pytest

import oracle
import pyref


def place_by_clusters(keys, last, missing, C, P, step):
    """keys/last after the refresh of resident ids; returns them after the
    inserts, placed cluster by cluster."""
    keys = keys.copy()
    last = last.copy()
    home = {k: pyref.home(k, C) for k in missing}
    slots = sorted(set(home.values()))
    n = len(slots)
    if n == 0:
        return keys, last
    # cut after slot i when the next occupied start slot (cyclically) is >= P away
    cut_after = [i for i in range(n) if n == 1 or (slots[(i + 1) % n] - slots[i]) % C >= P]
    if not cut_after:  # the windows chain all around the ring: one cluster
        clusters = [set(slots)]
    else:
        clusters = []
        for a, b in zip(cut_after, cut_after[1:] + [cut_after[0] + n]):
            clusters.append({slots[j % n] for j in range(a + 1, b + 1)})
    assert sum(len(c) for c in clusters) == n
    # clusters in an arbitrary order (reversed here): they must not interact
    for cl in reversed(clusters):
        for k in sorted(k for k in missing if home[k] in cl):
            window = [(home[k] + j) % C for j in range(P)]
            victim = min(window, key=lambda s: (last[s], s))
            keys[victim] = k
            last[victim] = step
    return keys, last


def run_case(seed, C, P, n_keys, batch, steps):
    rng = np.random.default_rng(seed)
    orc = oracle.OracleTable(C, 4, P)
    cut_cases = 0
    for t in range(steps):
        ids = rng.integers(0, n_keys, size=batch).astype(np.int64)
        e = rng.standard_normal((batch, 4)).astype(np.float32)
        keys0, last0, _ = orc.state()
        uniq, _ = oracle.dedup(ids)
        rc, rows, hit = orc.lookup(uniq)
        assert rc == 0
        last1 = last0.copy()
        last1[rows[hit != 0]] = t
        missing = [int(k) for k, h in zip(uniq, hit) if not h]
        want_keys, want_last = place_by_clusters(keys0, last1, missing, C, P, t)
        rc, _ = orc.writeback(ids, e, t)
        assert rc == 0
        keys2, last2, _ = orc.state()
        assert np.array_equal(keys2, want_keys), (seed, C, P, t)
        assert np.array_equal(last2, want_last), (seed, C, P, t)
        cut_cases += len(missing) * P < C and len(missing) > 1
    orc.close()
    return cut_cases


@pytest.mark.parametrize("C,P", [(8, 3), (16, 4), (37, 5), (64, 8), (97, 8), (128, 1), (200, 9)])
def test_cluster_placement_equals_sequential_insert(C, P):
    cut = 0
    for seed in range(40):
        rng = np.random.default_rng(1000 + seed)
        n_keys = int(rng.integers(C // 2 + 1, 4 * C))
        batch = int(rng.integers(1, max(2, C // 2)))
        cut += run_case(seed * 7 + C, C, P, n_keys, batch, steps=8)
    assert cut > 0  # steps where a cut exists and several clusters form
