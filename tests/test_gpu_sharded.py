"""Hash-owner sharding on the GPU against the sharded oracle.

* mpzch_owner_partition against its definition (a stable sort by the oracle's
  owner function; packed e rows), with ragged tiles, a device count, src_pos,
  one owner, the maximum number of owners, and an empty batch;
* mpzch_owner_combine against its definition (placement at batch positions,
  global rows, always-on concat, bad always-on rows);
* the whole sharded step (partition, first dedup, exchange, owner lookup /
  gather / Writeback, answers back, combine) for G = 1, 2, 3, 4 shards on one
  GPU -- G host threads with an in-process exchange, each rank on its own
  seeded id stream -- compared bit for bit with oracle.ShardedOracle: every
  rank's rows, hit and features, every shard's counters, and every shard's
  identity map, last-write steps and values.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from hashed_sparse_table_b200 import inputs
from gpu_harness import assert_bitwise, stats_dict, STATS_KEYS

pytestmark = pytest.mark.gpu

RANK_STRIDE = 1000  # id-stream offset between ranks (seed index t + 1000 * rank)


def _partition(ids, G, src_pos=None, dev_n=None, e=None):
    from hashed_sparse_table_b200 import binding
    dev = torch.device("cuda")
    n = ids.size
    ids_d = torch.from_numpy(ids).to(dev)
    ids_out = torch.full((n,), -7, dtype=torch.int64, device=dev)
    pos_out = torch.full((n,), -7, dtype=torch.int32, device=dev)
    counts = torch.full((G,), -7, dtype=torch.int64, device=dev)
    ws = torch.empty(binding.mpzch_owner_partition_workspace(n, G), dtype=torch.uint8, device=dev)
    e_d = e_out = None
    if e is not None:
        e_d = torch.from_numpy(e).to(dev)
        e_out = torch.full((n, e.shape[1]), float("nan"), dtype=torch.float32, device=dev)
    binding.mpzch_owner_partition(
        ids_d, G, ids_out, pos_out, counts, ws,
        src_pos=None if src_pos is None else torch.from_numpy(src_pos).to(dev),
        dev_n=None if dev_n is None else torch.tensor([dev_n], dtype=torch.int64, device=dev),
        e=e_d, e_out=e_out)
    return (ids_out.cpu().numpy(), pos_out.cpu().numpy(), counts.cpu().numpy(),
            None if e_out is None else e_out.cpu().numpy())


@pytest.mark.parametrize("n,G,use_src,dev_n,with_e,width", [
    (5000, 5, False, None, False, 16),     # ragged last tile
    (3 * 1024, 8, True, None, True, 16),   # whole tiles, src positions, e rows
    (7777, 3, True, 4321, True, 16),       # device count below n
    (2048, 1, False, None, True, 16),      # one owner: order unchanged
    (20000, 256, False, None, False, 16),  # maximum owners
    (1, 4, False, None, True, 16),
    (100, 4, False, 0, True, 16),          # device count 0
    (9000, 8, True, 8500, True, 516),      # rows of 129 vectors: a second, one-vector round
    (4100, 2, False, None, True, 1028),    # rows of 257 vectors
])
def test_partition_is_a_stable_sort_by_owner(n, G, use_src, dev_n, with_e, width):
    rng = np.random.default_rng(n + G)
    ids = inputs.zipf_keys(rng, 0.9, 50_000, n)
    src = rng.permutation(n).astype(np.int32) if use_src else None
    e = rng.standard_normal((n, width)).astype(np.float32) if with_e else None
    got_ids, got_pos, got_cnt, got_e = _partition(ids, G, src, dev_n, e)
    m = n if dev_n is None else min(dev_n, n)
    own = oracle.owners(ids[:m], G)
    order = np.argsort(own, kind="stable")
    want_pos = (src[:m] if use_src else np.arange(m, dtype=np.int32))[order]
    assert_bitwise(got_cnt, np.bincount(own, minlength=G).astype(np.int64), "counts")
    assert_bitwise(got_ids[:m], ids[:m][order], "ids_out")
    assert_bitwise(got_pos[:m], want_pos.astype(np.int32), "pos_out")
    assert np.all(got_ids[m:] == -7) and np.all(got_pos[m:] == -7)  # untouched past n_eff
    if with_e:
        assert_bitwise(got_e[:m], e[want_pos], "packed e rows")


def test_partition_of_an_empty_batch_clears_counts():
    from hashed_sparse_table_b200 import binding
    dev = torch.device("cuda")
    z = torch.empty(0, dtype=torch.int64, device=dev)
    counts = torch.full((6,), 9, dtype=torch.int64, device=dev)
    binding.mpzch_owner_partition(z, 6, z, torch.empty(0, dtype=torch.int32, device=dev), counts,
                                  torch.empty(0, dtype=torch.uint8, device=dev))
    assert counts.cpu().tolist() == [0] * 6


def test_partition_rejects_bad_arguments():
    from hashed_sparse_table_b200 import binding
    dev = torch.device("cuda")
    ids = torch.arange(10, dtype=torch.int64, device=dev)
    out = torch.empty(10, dtype=torch.int64, device=dev)
    pos = torch.empty(10, dtype=torch.int32, device=dev)
    cnt = torch.empty(300, dtype=torch.int64, device=dev)
    ws = torch.empty(4096, dtype=torch.uint8, device=dev)
    for G in (0, 257):
        with pytest.raises(binding.MpzchError):
            binding.mpzch_owner_partition(ids, G, out, pos, cnt, ws)
    with pytest.raises(binding.MpzchError):  # workspace too small
        binding.mpzch_owner_partition(ids, 4, out, pos, cnt, ws[:0])


@pytest.mark.parametrize("D,A,n", [(32, 8, 3000), (512, 128, 20000), (1024, 288, 5000),
                                   (4, 0, 777)])
def test_combine_places_answers_at_batch_positions(D, A, n):
    """Rows of one round of loads (10 and 160 vectors), of two (328 vectors:
    answer and always-on parts across the rounds), and without an always-on
    table; entries far more than warps (one-entry-deep pipeline)."""
    from hashed_sparse_table_b200 import binding
    dev = torch.device("cuda")
    rng = np.random.default_rng(11 + D)
    G, Cs = 4, 1000
    ids = rng.integers(0, 1 << 40, size=n, dtype=np.int64)
    got_ids, got_pos, _, _ = _partition(ids, G)
    recv_rows = rng.integers(-1, Cs, size=n).astype(np.int32)
    recv_feat = rng.standard_normal((n, D)).astype(np.float32)
    ao = rng.standard_normal((50, A)).astype(np.float32) if A else None
    aor = rng.integers(0, 50, size=n).astype(np.int32)
    aor[17] = 50  # out of range: zeros and BADAO
    rows = torch.full((n,), -9, dtype=torch.int32, device=dev)
    hit = torch.full((n,), 9, dtype=torch.uint8, device=dev)
    out = torch.full((n, D + A), float("nan"), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    T = lambda x: torch.from_numpy(x).to(dev)  # noqa: E731
    binding.mpzch_owner_combine(T(got_ids), T(got_pos), G, Cs, T(recv_rows), T(recv_feat), rows,
                                hit, out, T(ao) if A else None, T(aor) if A else None, status)
    own = oracle.owners(got_ids, G)
    want_rows = np.empty(n, np.int32)
    want_hit = np.empty(n, np.uint8)
    want_out = np.empty((n, D + A), np.float32)
    want_rows[got_pos] = np.where(recv_rows >= 0, own * Cs + recv_rows, -1)
    want_hit[got_pos] = recv_rows >= 0
    want_out[got_pos, :D] = recv_feat
    if A:
        ok = (aor >= 0) & (aor < 50)
        want_out[:, D:] = np.where(ok[:, None], ao[np.clip(aor, 0, 49)], 0.0)
    assert_bitwise(rows.cpu().numpy(), want_rows, "rows")
    assert_bitwise(hit.cpu().numpy(), want_hit, "hit")
    assert_bitwise(out.cpu().numpy(), want_out, "out")
    assert status.item() == (4 if A else 0)


def _rank_inputs(w, t, r):
    tt = t + RANK_STRIDE * r
    ids = inputs.step_ids(w, tt)
    e = inputs.step_e(w, tt)
    aor = inputs.author_rows(w, ids[:w.labeled])
    return ids, e, aor


def run_sharded(w, G):
    """Runs w.steps sharded steps on G emulated ranks; returns per-rank, per-step
    host copies of (rows, hit, out, stats) and the shards' final state."""
    from hashed_sparse_table_b200 import sharded
    group = sharded.LocalExchangeGroup(G)
    ao = inputs.author_table(w)
    results = [[None] * w.steps for _ in range(G)]
    finals = [None] * G
    errors = []

    def rank_main(r):
        try:
            shard = sharded.ShardedMpzch(w.capacity, w.dim, w.probes, group.member(r))
            dev = shard.device
            ao_d = None if ao is None else torch.from_numpy(ao).to(dev)
            for t in range(w.steps):
                ids, e, aor = _rank_inputs(w, t, r)
                rows, hit, out, st = shard.train_step(
                    torch.from_numpy(ids).to(dev), w.labeled, torch.from_numpy(e).to(dev), t,
                    ao_d, None if aor is None else torch.from_numpy(aor).to(dev))
                results[r][t] = (rows.cpu().numpy(), hit.cpu().numpy(), out.cpu().numpy(),
                                 stats_dict(st))
            k, l, m = shard.table.state()
            finals[r] = (k.cpu().numpy(), l.cpu().numpy(), m.cpu().numpy(), shard.table.status(),
                         int(shard.status.item()))
            shard.close()
        except BaseException as ex:  # noqa: BLE001 -- re-raised by the caller
            errors.append(ex)
            group.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    if errors:
        raise errors[0]
    return results, finals


SHARD_W = inputs.Workload("sharded_small", 3, capacity=1 << 11, dim=64, probes=8, steps=10,
                          labeled=900, pool=2700, zipf_alpha=0.9, zipf_keys=30_000,
                          ao_rows=1 << 12, ao_dim=16, ao_kind="mix")


@pytest.mark.parametrize("G", [1, 2, 3, 4])
def test_sharded_step_matches_sharded_oracle(G):
    w = SHARD_W
    results, finals = run_sharded(w, G)
    so = oracle.ShardedOracle(G, w.capacity, w.dim, w.probes)
    ao = inputs.author_table(w)
    evicted = 0
    for t in range(w.steps):
        batches = [_rank_inputs(w, t, r) for r in range(G)]
        for r, (ids, e, aor) in enumerate(batches):
            rc, orows, ohit, oout = so.lookup_gather(ids[:w.labeled], ao, aor)
            assert rc == 0
            rows, hit, out, _ = results[r][t]
            assert_bitwise(rows, orows, f"G={G} step {t} rank {r}: rows")
            assert_bitwise(hit, ohit, f"G={G} step {t} rank {r}: hit")
            assert_bitwise(out, oout, f"G={G} step {t} rank {r}: features")
        res = so.writeback([b[0] for b in batches], [b[1] for b in batches], t)
        for s, (rc, ost) in enumerate(res):
            assert rc == 0
            gst = results[s][t][3]
            for k in STATS_KEYS:
                if k == "n_ids" and G == 1:
                    # one shard: no first dedup, the table's Writeback sees the batch itself
                    assert gst[k] == int((batches[0][0] >= 0).sum()), (t, gst)
                    continue
                assert gst[k] == ost[k], (G, t, s, k, gst, ost)
            evicted += ost["n_evicted"]
    assert evicted > 0  # the workload fills the shards
    for s in range(G):
        keys, last, M, tstatus, cstatus = finals[s]
        ok, ol, _ = so.state(s)
        assert_bitwise(keys, ok, f"G={G} shard {s}: keys")
        assert_bitwise(last, ol, f"G={G} shard {s}: last")
        assert_bitwise(M, so.values(s), f"G={G} shard {s}: values")
        assert tstatus == 0 and cstatus == 0
    so.close()


def test_sharded_step_with_negative_ids():
    """Negative ids: the owner's lookup reports them as misses (bad-key status
    on the owner's table), the rank's first dedup skips them (bad-key status on
    the rank's own table), and every other output matches the sharded oracle."""
    from hashed_sparse_table_b200 import sharded
    w = SHARD_W.scaled(steps=3, labeled=300, pool=900)
    G = 2
    group = sharded.LocalExchangeGroup(G)
    ao = inputs.author_table(w)
    got = [[None] * w.steps for _ in range(G)]
    status = [None] * G
    errors = []

    def batch(t, r):
        ids, e, aor = _rank_inputs(w, t, r)
        ids = ids.copy()
        ids[5::97] = -1 - np.arange(ids[5::97].size)  # negative ids in both parts
        return ids, e, inputs.author_rows(w, np.maximum(ids[:w.labeled], 0))

    def rank_main(r):
        try:
            shard = sharded.ShardedMpzch(w.capacity, w.dim, w.probes, group.member(r))
            dev = shard.device
            ao_d = torch.from_numpy(ao).to(dev)
            for t in range(w.steps):
                ids, e, aor = batch(t, r)
                rows, hit, out, st = shard.train_step(
                    torch.from_numpy(ids).to(dev), w.labeled, torch.from_numpy(e).to(dev), t,
                    ao_d, torch.from_numpy(aor).to(dev))
                got[r][t] = (rows.cpu().numpy(), hit.cpu().numpy(), out.cpu().numpy(),
                             stats_dict(st))
            status[r] = shard.table.status()
            shard.close()
        except BaseException as ex:  # noqa: BLE001
            errors.append(ex)
            group.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    if errors:
        raise errors[0]
    so = oracle.ShardedOracle(G, w.capacity, w.dim, w.probes)
    for t in range(w.steps):
        batches = [batch(t, r) for r in range(G)]
        for r, (ids, e, aor) in enumerate(batches):
            _, orows, ohit, oout = so.lookup_gather(ids[:w.labeled], ao, aor)
            rows, hit, out, _ = got[r][t]
            assert_bitwise(rows, orows, f"step {t} rank {r}: rows")
            assert_bitwise(hit, ohit, f"step {t} rank {r}: hit")
            assert_bitwise(out, oout, f"step {t} rank {r}: features")
        res = so.writeback([b[0] for b in batches], [b[1] for b in batches], t)
        for s, (rc, ost) in enumerate(res):
            assert rc == 0
            for k in ("n_unique", "n_hit_unique", "n_inserted", "n_evicted", "n_dropped"):
                assert got[s][t][3][k] == ost[k], (t, s, k)
    from hashed_sparse_table_b200 import binding
    assert all(st_ & binding.MPZCH_STATUS_BADKEY for st_ in status)
    so.close()
