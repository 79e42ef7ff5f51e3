"""CUDA path vs CPU oracle, bit for bit, at sizes the oracle finishes in seconds.

Every case spans several 1024-id tiles and several thread blocks with a
ragged tail, and compares the lookup rows / hit mask, the fused gather
(cached branch + always-on concat), the Writeback counters and the whole table
state (keys, last-write steps, values) after every step.  Edge cases: empty
batches, bad ids and rows, non-power-of-two capacity, P = 1, P = C, P > 32,
windows wrapping past the last row, heavy eviction with dropped writes, both
insert paths (cluster placement, with its whole-ring fallback, long chains and
shared start slots; claim rounds run fully grid-wide, fully in the single-block
finisher or split between them), checkpoint/resume, and repeatability.
"""
import numpy as np
import pytest
import torch

import oracle
from hashed_sparse_table_b200 import inputs
from gpu_harness import assert_bitwise, make_pair, run_pair, snapshot_from_export, compare_state

pytestmark = pytest.mark.gpu

W = inputs.Workload
SCALED = {
    # a 1M-row-style stream at 1/64 scale: Zipf 1.1 + 15% fresh keys
    "c2_small": W("c2_small", 2, capacity=1 << 14, dim=512, probes=8, steps=20, labeled=3000,
                  pool=0, zipf_alpha=1.1, zipf_keys=300_000, fresh_frac=0.15),
    # multi-table: labeled + pool, author concat by mixed key (ragged sizes)
    "c3_small": W("c3_small", 3, capacity=1 << 13, dim=512, probes=8, steps=20, labeled=700,
                  pool=2900, zipf_alpha=0.9, zipf_keys=40_000, ao_rows=1 << 13, ao_dim=128,
                  ao_kind="mix"),
    # capacity stress: more distinct ids per step than rows, heavy eviction and drops
    "c4_stress": W("c4_stress", 4, capacity=1 << 12, dim=64, probes=8, steps=12, labeled=6000,
                   pool=0, zipf_alpha=1.2, zipf_keys=100_000, fresh_frac=0.2),
    "nonpow2": W("nonpow2", 6, capacity=3001, dim=32, probes=5, steps=10, labeled=2500, pool=0,
                 zipf_alpha=1.0001, zipf_keys=20_000, fresh_frac=0.1, ao_rows=700, ao_dim=4,
                 ao_kind="mod"),
    "p1_direct": W("p1_direct", 7, capacity=2048, dim=16, probes=1, steps=10, labeled=1500,
                   pool=0, zipf_alpha=1.05, zipf_keys=10_000),
    "p_eq_c": W("p_eq_c", 8, capacity=64, dim=8, probes=64, steps=20, labeled=100, pool=0,
                zipf_alpha=1.1, zipf_keys=500),
    "p40": W("p40", 9, capacity=997, dim=8, probes=40, steps=10, labeled=700, pool=0,
             zipf_alpha=0.95, zipf_keys=5_000),
    "tiny_table": W("tiny_table", 10, capacity=8, dim=4, probes=3, steps=30, labeled=40, pool=0,
                    zipf_alpha=1.1, zipf_keys=60),
}


def test_tiny_workload_bit_exact_every_step():
    run_pair(inputs.CFG1_TINY)


@pytest.mark.parametrize("name", list(SCALED))
def test_scaled_workloads_bit_exact_every_step(name):
    run_pair(SCALED[name])


@pytest.mark.parametrize("name", ["c2_small", "c3_small", "c4_stress", "nonpow2", "p_eq_c"])
def test_fused_train_step_bit_exact_every_step(name):
    run_pair(SCALED[name], fused_step=True)


@pytest.mark.parametrize("name", ["c2_small", "c3_small", "c4_stress", "nonpow2"])
def test_pipelined_train_steps_bit_exact(name):
    from gpu_harness import run_pipelined
    run_pipelined(SCALED[name])


@pytest.mark.parametrize("name", ["c3_small", "c4_stress"])
def test_pipelined_train_steps_with_claim_rounds_bit_exact(name):
    from gpu_harness import run_pipelined
    run_pipelined(SCALED[name], cluster=0)


def test_pipelined_cluster_placement_on_the_grid_bit_exact():
    """Pipelined steps where the grid-wide placement passes (not the whole-ring
    fallback) do the inserts."""
    from gpu_harness import run_pipelined
    run_pipelined(CLUSTERED["clus_p8"])


def test_pipelined_steps_then_other_calls_are_ordered():
    """Calls on the caller's stream after pipelined steps see the final table."""
    from gpu_harness import run_pipelined
    w = SCALED["c3_small"].scaled(steps=8)
    tbl, orc = run_pipelined(w)
    ids = inputs.step_ids(w, 100)
    rows, hit = tbl.lookup(torch.from_numpy(ids).cuda())
    _, orows, ohit = orc.lookup(ids)
    assert_bitwise(rows.cpu().numpy(), orows, "lookup after pipelined steps")


def test_fused_train_step_with_no_labeled_ids():
    w = SCALED["c2_small"].scaled(steps=4)
    from gpu_harness import make_pair
    tbl, orc = make_pair(w)
    for t in range(4):
        ids = inputs.step_ids(w, t)
        e = inputs.step_e(w, t)
        st = torch.zeros(7, dtype=torch.int64, device="cuda")
        tbl.train_step(torch.from_numpy(ids).cuda(), 0, torch.from_numpy(e).cuda(), t, stats=st)
        orc.writeback(ids, e, t)
    compare_state(tbl, orc, "no labeled ids")


@pytest.mark.parametrize("wide", [0, 1, 4, 64])
def test_insert_rounds_split_does_not_change_results(wide):
    r = run_pair(SCALED["c4_stress"], wide_rounds=wide, cluster=0)
    if wide >= 1:  # conflicts really happened (the single-block finisher counts as one round)
        assert max(s["n_rounds"] for s in r.stats) >= 2
    assert sum(s["n_dropped"] for s in r.stats) > 0


CLUSTERED = {
    # missing ids x P stay below C, so the grid-wide cluster placement runs;
    # enough misses per step that multi-key clusters are common
    "clus_p8": W("clus_p8", 11, capacity=1 << 15, dim=32, probes=8, steps=12, labeled=3000,
                 pool=0, zipf_alpha=0.9, zipf_keys=60_000, fresh_frac=0.3),
    "clus_p16": W("clus_p16", 12, capacity=1 << 14, dim=16, probes=16, steps=16, labeled=1200,
                  pool=0, zipf_alpha=0.9, zipf_keys=80_000, fresh_frac=0.5),
    "clus_p3_nonpow2": W("clus_p3_nonpow2", 13, capacity=30011, dim=16, probes=3, steps=12,
                         labeled=4000, pool=0, zipf_alpha=0.95, zipf_keys=60_000,
                         fresh_frac=0.3),
}


@pytest.mark.parametrize("name", list(CLUSTERED))
@pytest.mark.parametrize("cluster", [1, 0])
def test_cluster_placement_and_claim_rounds_bit_exact(name, cluster):
    w = CLUSTERED[name]
    r = run_pair(w, cluster=cluster)
    # the cluster placement really ran (not the whole-ring fallback) on most steps
    grid_wide = [s for s in r.stats if 0 < s["n_inserted"] and s["n_inserted"] * w.probes < w.capacity]
    assert len(grid_wide) >= w.steps // 2
    assert sum(s["n_evicted"] for s in r.stats) > 0


def _keys_with_home(C, slots, count_per_slot, start):
    # test-side hash (the published SplitMix64, as in the input generator) to
    # build keys whose start slots are chosen
    cand = np.arange(start, start + (1 << 22), dtype=np.int64)
    homes = (inputs.splitmix64_np(cand) % np.uint64(C)).astype(np.int64)
    out = []
    for s_, c in zip(slots, count_per_slot):
        ks = cand[homes == s_][:c]
        assert ks.size == c
        out.append(ks)
    return np.concatenate(out)


@pytest.mark.parametrize("fused", [False, True])
def test_cluster_placement_long_chains_and_shared_slots(fused):
    """Clusters beyond the 32 keys sorted in registers: a chain of 40 keys with
    start slots 2 apart that wraps past the last row, and 36 keys sharing one
    start slot (28 of them are evicted again in the same step)."""
    C, P, D = 1 << 16, 8, 16
    w = W("crafted", 14, capacity=C, dim=D, probes=P, steps=4, labeled=400, pool=0,
          zipf_alpha=1.0, zipf_keys=1000)
    rng = np.random.default_rng(5)
    batches = []
    for t in range(4):
        chain = _keys_with_home(C, [(C - 30 + 2 * i + (t % 2)) % C for i in range(40)], [1] * 40,
                                start=(t + 1) << 24)
        shared = _keys_with_home(C, [C // 2 + 3 * t], [36], start=(t + 9) << 24)
        other = rng.integers(1 << 40, 1 << 41, size=200, dtype=np.int64)
        repeat = batches[-1][:50] if batches else np.empty(0, np.int64)
        ids = np.concatenate([chain, shared, other, repeat])
        batches.append(ids[rng.permutation(ids.size)])
    r = run_pair(w, steps=4, ids_fn=lambda t: batches[t], fused_step=fused)
    for s in r.stats:
        assert s["n_inserted"] * P < C  # the grid-wide cluster path
    assert sum(s["n_dropped"] for s in r.stats) >= 4 * 28


@pytest.mark.parametrize("eta", [0.5, 0.1, 2.0 / 3.0, 0.0, 1.75])
@pytest.mark.parametrize("name", ["c3_small", "c4_stress"])
def test_learning_rate_writeback_bit_exact(name, eta):
    run_pair(SCALED[name], eta=eta, fused_step=True)


def test_learning_rate_rejects_non_finite():
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(64, 4, 2)
    for bad in (float("nan"), float("inf"), -float("inf")):
        with pytest.raises(binding.MpzchError):
            binding.mpzch_set_learning_rate(tbl.h, bad)


@pytest.mark.parametrize("name", ["c3_small", "c4_stress", "nonpow2"])
@pytest.mark.parametrize("fused", [False, True])
def test_values_in_host_memory_bit_exact(name, fused):
    from hashed_sparse_table_b200 import binding
    run_pair(SCALED[name], fused_step=fused, flags=binding.MPZCH_VALUES_IN_HOST_MEMORY)


def test_values_in_host_memory_pipelined_and_export():
    from hashed_sparse_table_b200 import binding
    from gpu_harness import run_pipelined
    w = SCALED["c3_small"]
    tbl, orc = run_pipelined(w, flags=binding.MPZCH_VALUES_IN_HOST_MEMORY)
    rows_d, cnt_d = tbl.select_written_since(w.steps - 10)
    n = int(cnt_d.item())
    orows = orc.select_written_since(w.steps - 10)
    q, s, k = tbl.export_int8(rows_d, n=w.capacity, dev_n=cnt_d)
    oq, os_, ok = orc.export_int8(orows)
    assert_bitwise(q[:n].cpu().numpy(), oq, "int8 export from host values")
    assert_bitwise(s[:n].cpu().numpy(), os_, "scales from host values")


def test_create_ex_rejects_unknown_flags():
    from hashed_sparse_table_b200 import binding
    with pytest.raises(binding.MpzchError):
        binding.mpzch_create_ex(64, 4, 2, 0x80)


def test_repeatable_bytes():
    w = SCALED["c3_small"].scaled(steps=6)
    a = run_pair(w)
    b = run_pair(w)
    for x, y in zip(a.tbl.state(), b.tbl.state()):
        assert torch.equal(x, y)


def test_checkpoint_resume_is_bit_identical():
    from hashed_sparse_table_b200 import binding
    w = SCALED["c2_small"].scaled(steps=12)
    full = run_pair(w, state_every=0)
    part = run_pair(w, steps=6, state_every=0)
    keys, last, M = (x.clone() for x in part.tbl.state())
    saved_step = binding.mpzch_get_last_step(part.tbl.h)
    part.tbl.close()
    tbl2, orc2 = make_pair(w)
    k2, l2, m2 = tbl2.state()
    k2.copy_(keys)
    l2.copy_(last)
    m2.copy_(M)
    binding.mpzch_set_last_step(tbl2.h, saved_step)
    ok, ol, ols = part.orc.state()
    orc2.set_state(ok, ol, ols)
    for r in range(w.capacity):
        orc2.set_row(r, part.orc.row(r))
    torch.cuda.synchronize()
    resumed = run_pair(w, steps=6, start=6, tbl=tbl2, orc=orc2, state_every=0)
    for x, y in zip(full.tbl.state(), resumed.tbl.state()):
        assert torch.equal(x, y)


# ------------------------------------------------------------------ dedup
@pytest.mark.parametrize("n", [0, 1, 5, 1023, 1024, 1025, 4097, 70_001])
def test_dedup_matches_oracle(n):
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(1024, 4, 2)
    rng = np.random.default_rng(n)
    ids = inputs.zipf_keys(rng, 1.1, 50_000, n)
    uniq, pos, cnt = tbl.dedup(torch.from_numpy(ids).cuda())
    ou, op = oracle.dedup(ids)
    c = int(cnt.item())
    assert c == ou.size
    assert_bitwise(uniq[:c].cpu().numpy(), ou, "uniq")
    assert_bitwise(pos[:c].cpu().numpy().astype(np.int64), op, "pos")
    # scratch hash is left clean: a second call gives the same answer
    uniq2, pos2, cnt2 = tbl.dedup(torch.from_numpy(ids).cuda())
    assert int(cnt2.item()) == c and torch.equal(uniq2[:c], uniq[:c])


def test_dedup_all_same_and_all_distinct():
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(1024, 4, 2)
    for ids in (np.full(5000, 7, np.int64), np.arange(5000, dtype=np.int64)[::-1].copy()):
        uniq, pos, cnt = tbl.dedup(torch.from_numpy(ids).cuda())
        ou, op = oracle.dedup(ids)
        c = int(cnt.item())
        assert_bitwise(uniq[:c].cpu().numpy(), ou, "uniq")
        assert_bitwise(pos[:c].cpu().numpy().astype(np.int64), op, "pos")


# ------------------------------------------------------------------ export + serving
def test_select_export_and_serve_match_oracle():
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"]
    r = run_pair(w, state_every=5)
    tbl, orc = r.tbl, r.orc
    since = w.steps - 10
    rows_d, cnt_d = tbl.select_written_since(since)
    orows = orc.select_written_since(since)
    n = int(cnt_d.item())
    assert n == orows.size
    assert_bitwise(rows_d[:n].cpu().numpy(), orows, "select rows")
    # export consumes the device count directly (no host round trip)
    q, s, k = tbl.export_int8(rows_d, n=w.capacity, dev_n=cnt_d)
    oq, os_, ok = orc.export_int8(orows)
    assert_bitwise(q[:n].cpu().numpy(), oq, "int8 q")
    assert_bitwise(s[:n].cpu().numpy(), os_, "scale")
    assert_bitwise(k[:n].cpu().numpy(), ok, "keys")
    sk, sq, ss = snapshot_from_export(w.capacity, w.dim, orows, oq, os_, ok)
    cand = inputs.zipf_keys(np.random.default_rng(1), 0.9, w.zipf_keys, 5000)
    cand[::97] = 10**12 + np.arange(cand[::97].size)  # never-seen ids
    rc, orow, ohit, oout = oracle.serve_gather(sk, w.capacity, w.probes, sq, ss, w.dim, cand)
    assert rc == 0
    dev = tbl.device
    out = torch.empty((cand.size, w.dim), dtype=torch.float32, device=dev)
    grow = torch.empty(cand.size, dtype=torch.int32, device=dev)
    ghit = torch.empty(cand.size, dtype=torch.uint8, device=dev)
    binding.mpzch_serve_gather(torch.from_numpy(sk).to(dev), w.probes, torch.from_numpy(sq).to(dev),
                               torch.from_numpy(ss).to(dev), torch.from_numpy(cand).to(dev),
                               grow, ghit, out)
    assert_bitwise(grow.cpu().numpy(), orow, "serve rows")
    assert_bitwise(ghit.cpu().numpy(), ohit, "serve hit")
    assert_bitwise(out.cpu().numpy(), oout, "serve features")
    assert 0 < ohit.mean() < 1


@pytest.mark.parametrize("D", [16, 128, 256, 512, 1024])
def test_export_edge_rows(D):
    """All-zero rows (scale 0), rows with a single large element, negative absmax
    (dims 128, 256, 512 and 1024 take the interleaved row exporter, others the
    generic one)."""
    from hashed_sparse_table_b200 import binding
    C = 64
    tbl = binding.MpzchTable(C, D, 4)
    orc = oracle.OracleTable(C, D, 4)
    _, _, M = tbl.state()
    rng = np.random.default_rng(3)
    vals = rng.standard_normal((C, D)).astype(np.float32)
    vals[0] = 0
    vals[1] = 0
    vals[1, 5] = -3e-38
    vals[2] = np.float32(127.0) * (np.arange(D, dtype=np.float32) - np.float32(D // 2))
    vals[3] = np.float32(1e30)
    vals[4, :] = np.float32(-0.0)
    M.copy_(torch.from_numpy(vals))
    for r in range(C):
        orc.set_row(r, vals[r])
    rows = np.arange(C, dtype=np.int32)
    q, s, k = tbl.export_int8(torch.from_numpy(rows).cuda())
    oq, os_, ok = orc.export_int8(rows)
    assert_bitwise(q.cpu().numpy(), oq, "q")
    assert_bitwise(s.cpu().numpy(), os_, "scale")
    # rows outside [0, C): zero codes, scale 0, key -1 and the bad-row status
    bad = np.array([3, -1, C, 5, 2**31 - 1], np.int32)
    q, s, k = tbl.export_int8(torch.from_numpy(bad).cuda())
    assert tbl.status() == binding.MPZCH_STATUS_BADROW
    ok_at = np.array([0, 3])
    oq, os_, _ = orc.export_int8(bad[ok_at])
    assert_bitwise(q.cpu().numpy()[ok_at], oq, "q of valid rows")
    assert_bitwise(s.cpu().numpy()[ok_at], os_, "scale of valid rows")
    for i in (1, 2, 4):
        assert not q[i].any() and s[i].item() == 0.0 and k[i].item() == -1


@pytest.mark.parametrize("D", [64, 128, 256, 512, 1024])
def test_export_near_half_integer_quotients(D):
    """Rows built so that x/scale lands on or within a few ulps of k + 1/2 (the
    rounding boundary), plus subnormal-scale rows: every int8 byte must match
    the oracle's IEEE division and round-half-even."""
    from hashed_sparse_table_b200 import binding
    C = 512
    tbl = binding.MpzchTable(C, D, 4)
    orc = oracle.OracleTable(C, D, 4)
    rng = np.random.default_rng(11)
    vals = np.empty((C, D), np.float32)
    for r in range(C):
        a = np.float32(10.0 ** rng.uniform(-30, 30)) if r % 8 else np.float32(127.0)
        if r % 61 == 0:
            a = np.float32(3e-42)  # subnormal absmax: subnormal scale
        sc = np.float32(a / np.float32(127.0))
        k = rng.integers(-127, 127, size=D).astype(np.float32)
        x = ((k + np.float32(0.5)) * sc).astype(np.float32)
        nudge = rng.integers(-3, 4, size=D)
        x = np.array([np.nextafter(v, np.float32(np.inf) if n > 0 else np.float32(-np.inf))
                      if n else v for v, n in zip(x, nudge)], np.float32)
        x[0] = a  # the absmax element
        vals[r] = x
    _, _, M = tbl.state()
    M.copy_(torch.from_numpy(vals))
    for r in range(C):
        orc.set_row(r, vals[r])
    rows = np.arange(C, dtype=np.int32)
    q, s, k = tbl.export_int8(torch.from_numpy(rows).cuda())
    oq, os_, ok = orc.export_int8(rows)
    assert_bitwise(s.cpu().numpy(), os_, "scale")
    assert_bitwise(q.cpu().numpy(), oq, "q near half-integers")


# ------------------------------------------------------------------ error paths and empties
def test_empty_calls_and_step_order():
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(256, 8, 4)
    dev = tbl.device
    empty_i = torch.empty(0, dtype=torch.int64, device=dev)
    rows, hit = tbl.lookup(empty_i)
    assert rows.numel() == 0
    st = torch.full((7,), 99, dtype=torch.int64, device=dev)
    tbl.writeback(empty_i, torch.empty((0, 8), device=dev), 0, st)
    assert st.sum().item() == 0
    with pytest.raises(binding.MpzchError) as ei:
        tbl.writeback(empty_i, torch.empty((0, 8), device=dev), 0, st)
    assert ei.value.code == binding.MPZCH_EINVAL
    ids = torch.tensor([5, 6], dtype=torch.int64, device=dev)
    tbl.writeback(ids, torch.ones((2, 8), device=dev), 3, st)
    with pytest.raises(binding.MpzchError):
        tbl.writeback(ids, torch.ones((2, 8), device=dev), 2, st)
    # misaligned e
    big = torch.ones(2 * 8 + 1, device=dev)
    with pytest.raises(binding.MpzchError):
        binding.mpzch_writeback(tbl.h, ids, big[1:].view(2, 8), 9, st)
    assert tbl.status() == 0


def test_bad_ids_set_status_and_are_skipped():
    w = inputs.Workload("bad", 11, capacity=512, dim=8, probes=4, steps=3, labeled=300, pool=0,
                        zipf_alpha=1.1, zipf_keys=2000)

    def ids_fn(t):
        ids = inputs.step_ids(w, t)
        ids[::37] = -7
        return ids
    tbl, orc = make_pair(w)
    dev = tbl.device
    for t in range(3):
        ids = ids_fn(t)
        e = inputs.step_e(w, t)
        ids_d = torch.from_numpy(ids).to(dev)
        rows, hit = tbl.lookup(ids_d)
        st = torch.zeros(7, dtype=torch.int64, device=dev)
        tbl.writeback(ids_d, torch.from_numpy(e).to(dev), t, st)
        rc, orows, ohit = orc.lookup(ids)
        rc2, ost = orc.writeback(ids, e, t)
        assert rc == oracle.ORC_EBADKEY and rc2 == oracle.ORC_EBADKEY
        assert_bitwise(rows.cpu().numpy(), orows, "rows")
        assert st[0].item() == ost["n_ids"] and st[1].item() == ost["n_unique"]
        assert tbl.status() & 1
    compare_state(tbl, orc, "after bad ids")
    assert tbl.status() == 0  # cleared by the read


def test_gather_bad_rows_set_status_and_give_zeros():
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(128, 8, 4)
    dev = tbl.device
    rows = torch.tensor([0, 500, -3, 7], dtype=torch.int32, device=dev)
    hit = torch.tensor([1, 1, 1, 0], dtype=torch.uint8, device=dev)
    ao = torch.arange(16 * 4, dtype=torch.float32, device=dev).view(16, 4)
    aor = torch.tensor([1, 2, 99, 3], dtype=torch.int32, device=dev)
    out = tbl.gather_fused(rows, hit, ao, aor)
    st = tbl.status()
    assert st & binding.MPZCH_STATUS_BADROW and st & binding.MPZCH_STATUS_BADAO
    o = out.cpu().numpy()
    assert (o[1:3, :8] == 0).all() and (o[2, 8:] == 0).all()
    assert (o[0, 8:] == np.arange(4, 8)).all()
    with pytest.raises(binding.MpzchError):  # ao_dim not a multiple of 4
        tbl.gather_fused(rows, hit, torch.zeros((4, 6), device=dev), aor)


def test_launch_counter_and_trace():
    from hashed_sparse_table_b200 import binding
    w = SCALED["c2_small"].scaled(steps=3)
    tbl, orc = make_pair(w)
    binding.mpzch_trace_enable(tbl.h, True)
    before = binding.mpzch_launch_count()
    run_pair(w, tbl=tbl, orc=orc, state_every=0)
    tr = binding.mpzch_trace_read(tbl.h)
    assert binding.mpzch_launch_count() > before
    for ph in ("lookup", "gather", "dedup", "insert", "writeback"):
        ms, launches = tr[ph]
        assert launches > 0 and ms > 0, (ph, tr[ph])


@pytest.mark.parametrize("C", [1, 7, 2048, 2049, 6000, 8193, 100_003, 1 << 20, (1 << 22) + 5])
def test_select_tiles_ragged_tails_and_repeated_calls(C):
    """The select over one tile, exactly one, one plus one row, many with a
    ragged tail, the 1M-row table and 4M rows (2049 tiles); several calls in a
    row on the same table (the per-tile marks and counts are rewritten by every
    call); rows chosen by every threshold from none to all.  Compared with the
    oracle and with the definition (ascending rows with a live key and
    last >= since)."""
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(C, 4, 1)
    orc = oracle.OracleTable(C, 4, 1, track_all=False)
    rng = np.random.default_rng(C)
    keys = rng.integers(0, 1 << 40, C, dtype=np.int64)
    last = rng.integers(-1, 100, C, dtype=np.int64)
    empty = rng.random(C) < 0.3
    keys[empty] = -1
    last[empty] = -1
    k_d, l_d, _ = tbl.state()
    k_d.copy_(torch.from_numpy(keys))
    l_d.copy_(torch.from_numpy(last))
    orc.set_state(keys, last, 99)
    for since in (-5, 0, 37, 99, 100, 37):
        rows_d, cnt_d = tbl.select_written_since(since)
        n = int(cnt_d.item())
        want = np.nonzero((keys != -1) & (last >= since))[0].astype(np.int32)
        assert n == want.size, (since, n, want.size)
        assert_bitwise(rows_d[:n].cpu().numpy(), want, f"select since {since}")
        assert_bitwise(rows_d[:n].cpu().numpy(), orc.select_written_since(since),
                       f"select since {since} vs oracle")
    assert tbl.status() == 0


# a table with room (missing ids x P < C, so the grid-wide placement passes run)
# whose flat id stream touches a large share of the rows every step: the whole
# window of some missing ids was written in the same step, so an id written
# earlier in the step is evicted again (its write-list entry is cancelled)
DROPS = W("drops_p2", 14, capacity=4096, dim=16, probes=2, steps=14, labeled=1500, pool=0,
          zipf_alpha=0.6, zipf_keys=5_000, fresh_frac=0.05)


@pytest.mark.parametrize("write_list", [1, 0])
@pytest.mark.parametrize("fused", [False, True])
def test_cluster_path_drops_with_both_write_list_builders(write_list, fused):
    """Evictions of ids written earlier in the same step on the grid-wide
    cluster path, with the write list emitted at re-probe and placement
    (cancelled entries) and with the separate list kernel: identical counters,
    rows, features and state, every step."""
    from hashed_sparse_table_b200 import binding
    r = run_pair(DROPS, fused_step=fused,
                 options={binding.MPZCH_OPT_WRITE_LIST: write_list})
    assert sum(s["n_dropped"] for s in r.stats) > 0
    assert max(s["n_inserted"] for s in r.stats) * DROPS.probes < DROPS.capacity


@pytest.mark.parametrize("name", ["c3_small", "c4_stress"])
def test_pipelined_steps_with_the_separate_write_list_kernel(name):
    from gpu_harness import run_pipelined
    from hashed_sparse_table_b200 import binding
    run_pipelined(SCALED[name], options={binding.MPZCH_OPT_WRITE_LIST: 0})


@pytest.mark.parametrize("wide", [0, 2])
@pytest.mark.parametrize("name", ["c3_small", "c4_stress"])
def test_fused_step_claim_rounds_lookup_fill(name, wide):
    """The train step's lookup comes from the re-probe; on the claim-round
    insert path a kernel of its own fills it, followed by 0 or 2 grid-wide
    rounds: rows, hit, features and state bit-exact every step."""
    run_pair(SCALED[name].scaled(steps=8), fused_step=True, cluster=0, wide_rounds=wide)


def test_fused_step_labeled_negative_ids():
    """Negative ids among the labeled positions of a train step: rows -1, hit 0,
    zero cached branch, the bad-key status, and the rest bit-exact."""
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"].scaled(steps=4)
    tbl, orc = make_pair(w)
    ao = inputs.author_table(w)
    ao_d = torch.from_numpy(ao).cuda()
    for t in range(w.steps):
        ids = inputs.step_ids(w, t).copy()
        ids[3::41] = -7
        e = inputs.step_e(w, t, rows=ids.size)
        lab = w.labeled
        aor = inputs.author_rows(w, np.maximum(ids[:lab], 0))
        st = torch.zeros(7, dtype=torch.int64, device="cuda")
        rows, hit, out = tbl.train_step(torch.from_numpy(ids).cuda(), lab, torch.from_numpy(e).cuda(),
                                        t, ao_d, torch.from_numpy(aor).cuda(), st)
        _, orows, ohit = orc.lookup(ids[:lab])
        oout = orc.gather_fused(orows, ohit, ao, aor)
        orc.writeback(ids, e, t)
        assert_bitwise(rows.cpu().numpy(), orows, f"step {t}: rows")
        assert_bitwise(hit.cpu().numpy(), ohit, f"step {t}: hit")
        assert_bitwise(out.cpu().numpy(), oout, f"step {t}: features")
        assert tbl.status() & binding.MPZCH_STATUS_BADKEY
    compare_state(tbl, orc, "after negative labeled ids")


def test_pipelined_steps_sharing_rows_and_hit_buffers():
    """Pipelined steps that reuse one rows/hit pair (each with its own fused
    output): a step's lookup fill must wait for the previous step's gather,
    which reads those buffers.  Every step's features and the final rows/hit
    and state match the oracle."""
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"].scaled(steps=10)
    tbl, orc = make_pair(w)
    dev = tbl.device
    ao = inputs.author_table(w)
    ao_d = torch.from_numpy(ao).to(dev)
    lab = w.labeled
    host = [(inputs.step_ids(w, t), inputs.step_e(w, t)) for t in range(w.steps)]
    aor = [inputs.author_rows(w, h[0][:lab]) for h in host]
    dev_in = [(torch.from_numpy(i).to(dev), torch.from_numpy(e).to(dev),
               torch.from_numpy(a).to(dev)) for (i, e), a in zip(host, aor)]
    rows = torch.empty(lab, dtype=torch.int32, device=dev)
    hit = torch.empty(lab, dtype=torch.uint8, device=dev)
    outs = [torch.empty((lab, w.dim + ao.shape[1]), dtype=torch.float32, device=dev)
            for _ in range(w.steps)]
    stats = [torch.empty(7, dtype=torch.int64, device=dev) for _ in range(w.steps)]
    ready = torch.cuda.Event()
    ready.record()
    for t in range(w.steps):
        ids_d, e_d, aor_d = dev_in[t]
        binding.mpzch_train_step(tbl.h, ids_d, lab, e_d, t, rows, hit, outs[t], ao_d, aor_d,
                                 stats[t], inputs_ready=ready)
    torch.cuda.synchronize()
    for t in range(w.steps):
        ids, e = host[t]
        _, orows, ohit = orc.lookup(ids[:lab])
        oout = orc.gather_fused(orows, ohit, ao, aor[t])
        orc.writeback(ids, e, t)
        assert_bitwise(outs[t].cpu().numpy(), oout, f"step {t}: features")
        if t == w.steps - 1:
            assert_bitwise(rows.cpu().numpy(), orows, "last rows")
            assert_bitwise(hit.cpu().numpy(), ohit, "last hit")
    compare_state(tbl, orc, "shared rows/hit buffers")
    assert tbl.status() == 0


@pytest.mark.parametrize("P,D,n", [(1, 16, 1), (8, 512, 7), (8, 512, 100_003), (40, 1024, 20_000),
                                   (8, 132, 50_001)])
def test_serve_gather_windows_widths_and_lengths(P, D, n):
    """Serving gather against the oracle on a snapshot whose keys sit in their
    windows (an oracle table filled by Writebacks) with arbitrary int8 codes
    and scales: one id, fewer ids than warps, many ids per warp (the
    one-id-deep pipeline), windows wider than a warp (P = 40), rows of 16, 132
    (33 vectors), 512 and 1024 (beyond the overlapped round) values; the
    candidates mix resident ids, never-seen ids and negative ids."""
    from hashed_sparse_table_b200 import binding
    C = 4096
    orc = oracle.OracleTable(C, 4, P, track_all=False)
    rng = np.random.default_rng(P * 1000 + D)
    seen = rng.choice(1 << 40, 6000, replace=False).astype(np.int64)
    for t in range(3):
        ids = seen[t * 2000:(t + 1) * 2000]
        orc.writeback(ids, rng.standard_normal((ids.size, 4)).astype(np.float32), t)
    keys, _, _ = orc.state()
    q = rng.integers(-127, 128, (C, D), dtype=np.int64).astype(np.int8)
    scale = (rng.random(C) * 0.02).astype(np.float32)
    scale[::17] = 0.0
    cand = seen[rng.integers(0, seen.size, n)]
    fresh = rng.random(n) < 0.2
    cand[fresh] = (1 << 41) + np.arange(int(fresh.sum()))  # never seen
    cand[6::13] = -3
    rc, orow, ohit, oout = oracle.serve_gather(keys, C, P, q, scale, D, cand)
    dev = torch.device("cuda", 0)
    rows = torch.empty(n, dtype=torch.int32, device=dev)
    hit = torch.empty(n, dtype=torch.uint8, device=dev)
    out = torch.empty((n, D), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    binding.mpzch_serve_gather(torch.from_numpy(keys).to(dev), P, torch.from_numpy(q).to(dev),
                               torch.from_numpy(scale).to(dev), torch.from_numpy(cand).to(dev),
                               rows, hit, out, status=status)
    assert_bitwise(rows.cpu().numpy(), orow, "serve rows")
    assert_bitwise(hit.cpu().numpy(), ohit, "serve hit")
    assert_bitwise(out.cpu().numpy(), oout, "serve features")
    assert int(status.item()) == (binding.MPZCH_STATUS_BADKEY if n > 6 else 0)
    if n > 100:
        assert 0 < ohit.mean() < 1
