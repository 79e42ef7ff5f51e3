"""Multi-rank plumbing of bench.py on CPU with the gloo backend (world size 2):
the whole-job aggregate sums units over ranks and takes the max time, and each
rank draws its own replica id stream."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        units, ms = bench.reduce_over_ranks(1000.0 * (rank + 1), 5.0 + 3.0 * rank,
                                            torch.device("cpu"))
        ids, _ = bench.host_step(0, rank)
        gathered = [torch.zeros(8, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(ids[:8].copy()))
        out[rank] = (units, ms, [g.tolist() for g in gathered])
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_reduce_over_ranks_and_replica_streams():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    for r in range(world):
        units, ms, streams = out[r]
        assert units == 3000.0  # 1000 + 2000
        assert ms == 8.0        # max(5, 8)
        assert streams[0] != streams[1]  # replicas draw different id streams


def test_reduce_over_ranks_without_process_group_is_identity():
    import bench
    assert bench.reduce_over_ranks(7.0, 2.5, torch.device("cpu")) == (7.0, 2.5)
