"""Hash-owner sharding of the table over G ranks, one shard per rank.

Memory Layer section 2 shards the table across devices and keeps the
distributed lookup's all-to-all path; MTGR (section 3.3, Embedding Lookup)
exchanges ids all-to-all between devices and dedups them twice, before and
after the exchange.  Key k lives in shard owner(k) = (splitmix64(k) >> 32)
mod G; global row of shard s, local row r = s * shard_capacity + r.

One step on every rank (ranks take the same collective steps in the same
order):
  1. partition the labeled ids by owner (kernel), dedup the whole batch on
     the rank (kernel) and partition the distinct ids by owner, packing their
     e rows into the send buffer (kernel);
  2. exchange segment sizes, then ids and e rows, all-to-all;
  3. as owner: lookup + gather of the received labeled ids on the table as it
     was before the step, then the Writeback of the received distinct ids
     (which dedups again across ranks: ranks arrive in rank order);
  4. send the lookup answers back all-to-all and combine them at their batch
     positions with the rank's always-on rows (kernel).

prepare() does step 1 and starts the exchange of segment sizes (an
all-to-all whose result is copied to pinned host memory asynchronously);
finish() reads the sizes on the host and does the rest.  A caller that
issues step t+1's prepare before step t's finish (every rank in the same
order) never makes the host wait for the GPU in the middle of a step;
train_step() is prepare + finish.

Every step of the path runs in the library's kernels; this module only moves
segments between ranks: torch.distributed ``all_to_all_single`` (NCCL on the
GPUs), or ``LocalExchangeGroup`` for G shards on one GPU in one process.
"""
from __future__ import annotations

import threading
from typing import List, Optional

import torch


class DistExchange:
    """All-to-all between the ranks of a torch.distributed process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def sizes(self, send: torch.Tensor) -> torch.Tensor:
        """send: int64 [G, k] on this rank's device, row g for rank g.  Returns,
        on the host, [2, G, k]: what this rank sends and what it receives."""
        return self.sizes_wait(self.sizes_async(send))

    def sizes_async(self, send: torch.Tensor):
        """Starts the exchange of `send` and its copy to pinned host memory;
        sizes_wait returns the host tensor once the copy has landed."""
        recv = torch.empty_like(send)
        self.dist.all_to_all_single(recv, send, group=self.group)
        both = torch.stack([send, recv])
        if not both.is_cuda:
            return both, None
        host = torch.empty(both.shape, dtype=both.dtype, pin_memory=True)
        host.copy_(both, non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        return host, ev

    @staticmethod
    def sizes_wait(handle) -> torch.Tensor:
        host, ev = handle
        if ev is not None:
            ev.synchronize()
        return host

    def all_to_all(self, send: torch.Tensor, send_splits: List[int],
                   recv_splits: List[int]) -> torch.Tensor:
        out = send.new_empty((sum(recv_splits),) + tuple(send.shape[1:]))
        self.dist.all_to_all_single(out, send[:sum(send_splits)], recv_splits, send_splits,
                                    group=self.group)
        return out


class LocalExchangeGroup:
    """G ranks emulated by G host threads of one process: each exchange is a
    rendezvous of all G threads; rank r receives the segments addressed to it
    in rank order.  The threads' kernels never wait on one another -- every
    rank's work is complete (stream synchronised) before it is handed over."""

    def __init__(self, world: int, timeout: float = 300.0, cuda: bool = True):
        self.world, self.cuda = world, cuda
        self.barrier = threading.Barrier(world, timeout=timeout)
        self.slots = [None] * world

    def member(self, rank: int) -> "LocalExchange":
        return LocalExchange(self, rank)

    def abort(self):
        self.barrier.abort()


class LocalExchange:
    def __init__(self, group: LocalExchangeGroup, rank: int):
        self.g, self.rank, self.world = group, rank, group.world

    def _sync(self):
        if self.g.cuda:
            torch.cuda.current_stream().synchronize()

    def _swap(self, item):
        self._sync()
        self.g.slots[self.rank] = item
        self.g.barrier.wait()
        got = list(self.g.slots)
        return got

    def _done(self):
        self._sync()
        self.g.barrier.wait()

    def sizes(self, send: torch.Tensor) -> torch.Tensor:
        got = self._swap(send.cpu())
        recv = torch.stack([got[src][self.rank] for src in range(self.world)])
        out = torch.stack([got[self.rank], recv])
        self._done()
        return out

    def sizes_async(self, send: torch.Tensor):
        return self.sizes(send), None

    @staticmethod
    def sizes_wait(handle) -> torch.Tensor:
        return handle[0]

    def all_to_all(self, send: torch.Tensor, send_splits: List[int],
                   recv_splits: List[int]) -> torch.Tensor:
        got = self._swap((send, send_splits))
        parts = []
        for src in range(self.world):
            buf, splits = got[src]
            lo = sum(splits[:self.rank])
            parts.append(buf[lo:lo + splits[self.rank]])
            assert splits[self.rank] == recv_splits[src]
        out = torch.cat(parts) if parts else send.new_empty((0,) + tuple(send.shape[1:]))
        self._done()
        return out


class ShardedMpzch:
    """This rank's shard and the step that routes ids to their owners."""

    def __init__(self, shard_capacity: int, dim: int, probes: int, exchange, flags: int = 0):
        from . import binding  # the CUDA library; raises ImportError when it is not built
        self.binding = binding
        self.G, self.rank, self.ex = exchange.world, exchange.rank, exchange
        if not 1 <= self.G <= binding.MPZCH_MAX_OWNERS:
            raise ValueError(f"{self.G} shards; at most {binding.MPZCH_MAX_OWNERS}")
        self.capacity, self.dim, self.probes = shard_capacity, dim, probes
        self.table = binding.MpzchTable(shard_capacity, dim, probes, flags=flags)
        self.device = self.table.device
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws = torch.empty(0, dtype=torch.uint8, device=self.device)

    def close(self):
        self.table.close()

    def _workspace(self, n: int) -> torch.Tensor:
        need = self.binding.mpzch_owner_partition_workspace(n, self.G)
        if self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def train_step(self, ids: torch.Tensor, n_labeled: int, e: torch.Tensor, step: int,
                   ao_table: Optional[torch.Tensor] = None, ao_rows: Optional[torch.Tensor] = None,
                   rows=None, hit=None, out=None, stats=None, trace: Optional[dict] = None):
        """Rows (global), hit and fused features of the labeled ids (read
        before this step's Writeback), and this shard's Writeback counters.

        With one shard every id is owned here and global rows are local rows,
        so the step is the table's own train step: no partition, exchange or
        combine, and no host read of segment sizes.  The counters are then
        those of that step; they differ from a multi-shard step's only in
        n_ids, which counts the batch's valid ids (no first dedup ran)."""
        return self.finish(self.prepare(ids, n_labeled, e), step, ao_table, ao_rows, rows, hit,
                           out, stats, trace)

    def prepare(self, ids: torch.Tensor, n_labeled: int, e: torch.Tensor,
                inputs_ready=None) -> "Prepared":
        """Steps 1-2a of a sharded step: the partitions by owner (labeled ids;
        distinct ids with their e rows packed) and the start of the segment-
        size exchange.  Issuing the next step's prepare before this step's
        finish lets the sizes reach the host while this step runs, so the host
        never waits for the GPU in the middle of a step.  Every rank must issue
        prepares and finishes in the same order (they are collectives).
        inputs_ready (a CUDA event recorded after ids and e were written) lets a
        one-shard step run pipelined like the table's own train step."""
        if self.G == 1:
            return Prepared(ids=ids, n_labeled=n_labeled, e=e, inputs_ready=inputs_ready)
        binding = self.binding
        G, dev, D = self.G, self.device, self.dim
        n = ids.numel()
        lab = ids[:n_labeled]
        counts = torch.empty((2, G), dtype=torch.int64, device=dev)
        ws = self._workspace(max(n, n_labeled))  # both partitions run in order on one stream
        l_ids = torch.empty(n_labeled, dtype=torch.int64, device=dev)
        l_pos = torch.empty(n_labeled, dtype=torch.int32, device=dev)
        binding.mpzch_owner_partition(lab, G, l_ids, l_pos, counts[0], ws)
        uniq, upos, ucnt = self.table.dedup(ids)
        w_ids = torch.empty(n, dtype=torch.int64, device=dev)
        w_pos = torch.empty(n, dtype=torch.int32, device=dev)
        w_e = torch.empty((n, D), dtype=torch.float32, device=dev)
        binding.mpzch_owner_partition(uniq, G, w_ids, w_pos, counts[1], ws, src_pos=upos,
                                      dev_n=ucnt, e=e, e_out=w_e)
        return Prepared(ids=ids, n_labeled=n_labeled, e=e, l_ids=l_ids, l_pos=l_pos, w_ids=w_ids,
                        w_e=w_e, sizes=self.ex.sizes_async(counts.t().contiguous()))

    def finish(self, prep: "Prepared", step: int, ao_table: Optional[torch.Tensor] = None,
               ao_rows: Optional[torch.Tensor] = None, rows=None, hit=None, out=None, stats=None,
               trace: Optional[dict] = None):
        """Steps 2b-4 of a sharded step prepared by prepare()."""
        binding = self.binding
        G, dev, D = self.G, self.device, self.dim
        n_labeled = prep.n_labeled
        width = D + (0 if ao_table is None else ao_table.shape[1])
        rows = torch.empty(n_labeled, dtype=torch.int32, device=dev) if rows is None else rows
        hit = torch.empty(n_labeled, dtype=torch.uint8, device=dev) if hit is None else hit
        out = torch.empty((n_labeled, width), dtype=torch.float32, device=dev) if out is None else out
        stats = torch.empty(7, dtype=torch.int64, device=dev) if stats is None else stats
        if G == 1:
            self.table.train_step(prep.ids, n_labeled, prep.e, step, ao_table, ao_rows, stats,
                                  inputs_ready=prep.inputs_ready, rows=rows, hit=hit, out=out)
            if trace is not None:
                trace["sent_lookup"] = trace["sent_writeback"] = trace["recv_writeback"] = 0
            return rows, hit, out, stats
        # 2b. segment sizes on the host, then ids and e rows
        sz = self.ex.sizes_wait(prep.sizes).tolist()  # [send|recv][peer][lookup|wb]
        s_l = [sz[0][g][0] for g in range(G)]
        r_l = [sz[1][g][0] for g in range(G)]
        s_w = [sz[0][g][1] for g in range(G)]
        r_w = [sz[1][g][1] for g in range(G)]
        r_lids = self.ex.all_to_all(prep.l_ids, s_l, r_l)
        r_wids = self.ex.all_to_all(prep.w_ids, s_w, r_w)
        r_we = self.ex.all_to_all(prep.w_e, s_w, r_w)
        # 3. owner: lookup + gather before the Writeback
        r_rows, r_hit = self.table.lookup(r_lids)
        r_feat = self.table.gather_fused(r_rows, r_hit)
        self.table.writeback(r_wids, r_we, step, stats)
        # 4. answers back in send order, placed at their batch positions
        b_rows = self.ex.all_to_all(r_rows, r_l, s_l)
        b_feat = self.ex.all_to_all(r_feat, r_l, s_l)
        binding.mpzch_owner_combine(prep.l_ids, prep.l_pos, G, self.capacity, b_rows, b_feat, rows,
                                    hit, out, ao_table, ao_rows, self.status)
        if trace is not None:
            trace["sent_lookup"] = sum(s_l)
            trace["sent_writeback"] = sum(s_w)
            trace["recv_writeback"] = sum(r_w)
        return rows, hit, out, stats


class Prepared:
    """The partitioned buffers and the pending segment sizes of one sharded step."""

    def __init__(self, ids, n_labeled, e, l_ids=None, l_pos=None, w_ids=None, w_e=None,
                 sizes=None, inputs_ready=None):
        self.ids, self.n_labeled, self.e = ids, n_labeled, e
        self.l_ids, self.l_pos, self.w_ids, self.w_e = l_ids, l_pos, w_ids, w_e
        self.sizes, self.inputs_ready = sizes, inputs_ready
