"""The sharded step's orchestration across two real ranks, on the CPU.

ShardedMpzch.train_step runs unchanged with DistExchange over two gloo
processes (world size 2).  The CUDA library is replaced by test doubles: the
owner partition and the combine written from their definitions, and each
rank's shard an oracle table behind the same tensor-in / tensor-out calls.  So
this checks what only a multi-rank run exercises -- segment sizes exchanged
and read back in the right order, ids / e rows / answers sent to and received
from the right peers, answers put back at the right batch positions -- against
oracle.ShardedOracle, which routes by its own plain rule.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

G = 2
C_S, D, P = 64, 8, 4
STEPS, BATCH, LABELED, N_KEYS = 5, 60, 25, 400
AO_ROWS, AO_DIM = 32, 4


def rank_batch(t, r):
    rng = np.random.default_rng(100 * t + r)
    ids = (rng.pareto(1.1, size=BATCH) * 11).astype(np.int64) % N_KEYS
    e = rng.standard_normal((BATCH, D)).astype(np.float32)
    aor = (ids[:LABELED] % AO_ROWS).astype(np.int32)
    return ids, e, aor


def ao_table():
    return np.random.default_rng(7).standard_normal((AO_ROWS, AO_DIM)).astype(np.float32)


class FakeBinding:
    """Partition and combine by their definitions (see include/mpzch.h)."""
    MPZCH_MAX_OWNERS = 256

    @staticmethod
    def mpzch_owner_partition_workspace(n, n_owners):
        return 0

    @staticmethod
    def mpzch_owner_partition(ids, n_owners, ids_out, pos_out, counts, workspace, src_pos=None,
                              dev_n=None, e=None, e_out=None):
        n = ids.numel() if dev_n is None else int(dev_n.reshape(-1)[0])
        k = ids[:n].numpy()
        own = oracle.owners(k, n_owners)
        order = np.argsort(own, kind="stable")
        src = np.arange(n) if src_pos is None else src_pos[:n].numpy().astype(np.int64)
        ids_out[:n] = torch.from_numpy(k[order])
        pos_out[:n] = torch.from_numpy(src[order].astype(np.int32))
        counts.copy_(torch.from_numpy(np.bincount(own, minlength=n_owners).astype(np.int64)))
        if e is not None:
            e_out[:n] = e[torch.from_numpy(src[order])]

    @staticmethod
    def mpzch_owner_combine(send_ids, pos, n_owners, shard_capacity, recv_rows, recv_feat, rows, hit,
                            out, ao_table=None, ao_rows=None, status=None, stream=None, n=None):
        n = send_ids.numel() if n is None else n
        own = oracle.owners(send_ids[:n].numpy(), n_owners).astype(np.int64)
        p = pos[:n].numpy().astype(np.int64)
        r = recv_rows[:n].numpy().astype(np.int64)
        rows[p] = torch.from_numpy(np.where(r >= 0, own * shard_capacity + r, -1).astype(np.int32))
        hit[p] = torch.from_numpy((r >= 0).astype(np.uint8))
        out[p, :recv_feat.shape[1]] = recv_feat[:n]
        if ao_table is not None:
            out[:, recv_feat.shape[1]:] = ao_table[ao_rows.long()]


class FakeTable:
    """One shard: the oracle table behind the calls ShardedMpzch makes."""

    def __init__(self, capacity, dim, probes):
        self.orc = oracle.OracleTable(capacity, dim, probes)

    def dedup(self, ids):
        n = ids.numel()
        uniq, pos = oracle.dedup(ids.numpy())
        u = torch.zeros(n, dtype=torch.int64)
        p = torch.zeros(n, dtype=torch.int32)
        u[:uniq.size] = torch.from_numpy(uniq)
        p[:pos.size] = torch.from_numpy(pos.astype(np.int32))
        return u, p, torch.tensor([uniq.size], dtype=torch.int64)

    def lookup(self, ids):
        rc, rows, hit = self.orc.lookup(ids.numpy())
        assert rc == 0
        return torch.from_numpy(rows), torch.from_numpy(hit)

    def gather_fused(self, rows, hit):
        return torch.from_numpy(self.orc.gather_fused(rows.numpy(), hit.numpy()))

    def writeback(self, ids, e, step, stats=None):
        rc, st = self.orc.writeback(ids.numpy(), e.numpy(), step)
        assert rc == 0
        keys = ("n_ids", "n_unique", "n_hit_unique", "n_inserted", "n_evicted", "n_dropped")
        stats[:6] = torch.tensor([st[k] for k in keys], dtype=torch.int64)


def _worker(rank, world, port, out, lookahead=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from hashed_sparse_table_b200.sharded import DistExchange, ShardedMpzch
        sh = ShardedMpzch.__new__(ShardedMpzch)  # the library-free parts of a shard
        sh.binding = FakeBinding
        sh.ex = DistExchange()
        sh.G, sh.rank = sh.ex.world, sh.ex.rank
        sh.capacity, sh.dim, sh.probes = C_S, D, P
        sh.table = FakeTable(C_S, D, P)
        sh.device = torch.device("cpu")
        sh.status = torch.zeros(1, dtype=torch.int32)
        sh._ws = torch.empty(0, dtype=torch.uint8)
        ao = torch.from_numpy(ao_table())
        res = []

        def prep(t):
            ids, e, _ = rank_batch(t, rank)
            return sh.prepare(torch.from_numpy(ids), LABELED, torch.from_numpy(e))

        nxt = prep(0) if lookahead else None
        for t in range(STEPS):
            ids, e, aor = rank_batch(t, rank)
            if lookahead:  # step t+1 is prepared (sizes exchanged) before step t finishes
                cur = nxt
                nxt = prep(t + 1) if t + 1 < STEPS else None
                rows, hit, feats, st = sh.finish(cur, t, ao, torch.from_numpy(aor))
            else:
                rows, hit, feats, st = sh.train_step(torch.from_numpy(ids), LABELED,
                                                     torch.from_numpy(e), t, ao,
                                                     torch.from_numpy(aor))
            res.append((rows.numpy().copy(), hit.numpy().copy(), feats.numpy().copy(),
                        st.numpy().copy()))
        out[rank] = (res, sh.table.orc.state()[0], sh.table.orc.values())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("lookahead", [False, True])
def test_sharded_step_over_two_gloo_ranks_matches_the_sharded_oracle(lookahead):
    """train_step per step, and prepare(t+1) issued before finish(t)."""
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(G, _free_port(), out, lookahead), nprocs=G,
                       start_method="spawn", join=True)
    so = oracle.ShardedOracle(G, C_S, D, P)
    ao = ao_table()
    evicted = 0
    for t in range(STEPS):
        batches = [rank_batch(t, r) for r in range(G)]
        for r, (ids, e, aor) in enumerate(batches):
            _, orows, ohit, oout = so.lookup_gather(ids[:LABELED], ao, aor)
            rows, hit, feats, _ = out[r][0][t]
            assert np.array_equal(rows, orows), (t, r)
            assert np.array_equal(hit, ohit), (t, r)
            assert np.array_equal(feats.view(np.uint32), oout.view(np.uint32)), (t, r)
        res = so.writeback([b[0] for b in batches], [b[1] for b in batches], t)
        for s, (rc, ost) in enumerate(res):
            assert rc == 0
            st = out[s][0][t][3]
            assert list(st[:6]) == [ost[k] for k in ("n_ids", "n_unique", "n_hit_unique",
                                                     "n_inserted", "n_evicted", "n_dropped")]
            evicted += ost["n_evicted"]
    for s in range(G):
        keys, vals = out[s][1], out[s][2]
        assert np.array_equal(keys, so.state(s)[0])
        assert np.array_equal(vals.view(np.uint32), so.values(s).view(np.uint32))
    assert evicted > 0
    so.close()
