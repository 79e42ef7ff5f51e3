"""The all-to-all exchange of the sharded step on CPU (no GPU needed).

Two gloo ranks (world size 2) route owner-sorted segments of ids and e rows
through DistExchange -- segment sizes first, then 1-D ids and 2-D rows, with
empty segments in both directions -- and each rank must receive exactly the
segments addressed to it, in rank order.  The in-process exchange used for G
shards on one GPU must deliver the same bytes for the same sends.
"""
import datetime
import os
import socket
import threading

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

G = 2
D = 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_send(rank, case):
    """Owner-sorted ids / rows a rank sends, and its per-owner segment sizes."""
    rng = np.random.default_rng(100 * case + rank)
    n = [700, 0, 333][case] if rank == 0 else [450, 210, 0][case]
    ids = rng.integers(0, 1 << 40, size=n, dtype=np.int64)
    if case == 1 and rank == 1:  # rank 1 sends only to itself
        ids = ids[oracle.owners(ids, G) == 1]
    own = oracle.owners(ids, G)
    order = np.argsort(own, kind="stable")
    rows = rng.standard_normal((ids.size, D)).astype(np.float32)
    return ids[order], rows[order], np.bincount(own, minlength=G).astype(np.int64)


def expected_recv(rank, case):
    ids, rows = [], []
    for src in range(G):
        s_ids, s_rows, cnt = rank_send(src, case)
        lo = int(cnt[:rank].sum())
        ids.append(s_ids[lo:lo + cnt[rank]])
        rows.append(s_rows[lo:lo + cnt[rank]])
    return np.concatenate(ids), np.concatenate(rows)


def run_exchange(ex, rank, case):
    ids, rows, cnt = rank_send(rank, case)
    sz = ex.sizes(torch.from_numpy(np.stack([cnt, cnt * 0 + 1], 1))).tolist()
    send = [sz[0][g][0] for g in range(G)]
    recv = [sz[1][g][0] for g in range(G)]
    assert [sz[1][g][1] for g in range(G)] == [1] * G
    r_ids = ex.all_to_all(torch.from_numpy(ids), send, recv)
    r_rows = ex.all_to_all(torch.from_numpy(rows), send, recv)
    return r_ids.numpy().copy(), r_rows.numpy().copy()


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from hashed_sparse_table_b200.sharded import DistExchange
        ex = DistExchange()
        assert ex.world == world and ex.rank == rank
        out[rank] = [run_exchange(ex, rank, case) for case in range(3)]
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_dist_exchange_delivers_owner_segments_in_rank_order():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(G, port, out), nprocs=G, start_method="spawn", join=True)
    for rank in range(G):
        for case in range(3):
            got_ids, got_rows = out[rank][case]
            want_ids, want_rows = expected_recv(rank, case)
            assert np.array_equal(got_ids, want_ids), (rank, case)
            assert np.array_equal(got_rows.view(np.uint32), want_rows.view(np.uint32)), (rank, case)


def test_local_exchange_matches_the_definition():
    from hashed_sparse_table_b200.sharded import LocalExchangeGroup

    group = LocalExchangeGroup(G, timeout=60, cuda=False)
    res = [None] * G
    errors = []

    def main(r):
        try:
            res[r] = [run_exchange(group.member(r), r, case) for case in range(3)]
        except BaseException as e:  # noqa: BLE001
            errors.append(e)
            group.abort()

    th = [threading.Thread(target=main, args=(r,)) for r in range(G)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    for rank in range(G):
        for case in range(3):
            want_ids, want_rows = expected_recv(rank, case)
            assert np.array_equal(res[rank][case][0], want_ids)
            assert np.array_equal(res[rank][case][1].view(np.uint32), want_rows.view(np.uint32))
