"""CUDA path vs CPU oracle at the full workload sizes, through the same calls
and launch configuration the benchmark times: mpzch_reserve for the batch, then
one pipelined mpzch_train_step per step (lookup -> fused gather -> Writeback,
with an inputs-ready event so a step's row map overlaps the previous step's
row update), the item-tower target pool resident on the device.

* 1M rows x 512, 8 probes, 100 steps of 65,536 ids (Zipf 1.1 over 20M + 15%
  fresh): every lookup row / hit and Writeback counter, the identity map and
  last-write steps every 10 steps, gathered features (all rows every 10th
  step, a sample otherwise), and all 2 GiB of values at the end.
* multi-table (the benchmark's workload): same checks, plus the always-on
  author concat; then the serving/export workload on its final state: rows
  written in the last 50 steps, their int8 export, and the serving gather of
  4,096 x 1,024 candidates in 512-request chunks, all compared in full.
* 16M rows x 512 (32 GiB): identity map and last-write steps every 20 steps
  and at the end, every counter and lookup, and the values: all 32 GiB at the
  end (compared in 1M-row chunks) when the host has the memory for the
  oracle's full table, otherwise every 64th row (262,144 rows), in which case
  every gathered hit on such a row is checked too.

Inputs are the same seeded generators as everywhere; each workload's pool of
item-tower target batches is uploaded once.
"""
import numpy as np
import pytest
import torch

import oracle
from hashed_sparse_table_b200 import inputs
from gpu_harness import assert_bitwise, bits, stats_dict, STATS_KEYS, snapshot_from_export

pytestmark = pytest.mark.gpu


class Pool:
    """Host + device copies of a workload's item-tower target batches."""

    def __init__(self, w, dev):
        self.host = [inputs.step_e(w, t) for t in range(inputs.E_POOL)]
        self.dev = [torch.from_numpy(x).to(dev) for x in self.host]

    def __call__(self, t):
        return self.host[t % inputs.E_POOL], self.dev[t % inputs.E_POOL]


def run_full(w, check_state_every, full_gather_every, value_rows=None, gather_sample=2048,
             chunk=10):
    """Steps are issued as the benchmark issues them: pipelined mpzch_train_step
    calls with an inputs-ready event, `chunk` steps at a time with their own
    output buffers; then each step is checked against the oracle in order."""
    from hashed_sparse_table_b200 import binding
    dev = torch.device("cuda", torch.cuda.current_device())
    tbl = binding.MpzchTable(w.capacity, w.dim, w.probes)
    binding.mpzch_reserve(tbl.h, w.batch)
    orc = oracle.OracleTable(w.capacity, w.dim, w.probes, track_all=value_rows is None)
    if value_rows is not None:
        orc.track_rows(value_rows)
        tracked = np.zeros(w.capacity, bool)
        tracked[value_rows] = True
    pool = Pool(w, dev)
    ao = inputs.author_table(w)
    ao_d = torch.from_numpy(ao).to(dev) if ao is not None else None
    lab = w.labeled
    width = w.dim + (0 if ao is None else ao.shape[1])
    rng = np.random.default_rng(99)
    assert check_state_every % chunk == 0
    for c0 in range(0, w.steps, chunk):
        steps = list(range(c0, min(c0 + chunk, w.steps)))
        host = {t: inputs.step_ids(w, t) for t in steps}
        aor = {t: inputs.author_rows(w, host[t][:lab]) for t in steps}
        dev_ids = {t: torch.from_numpy(host[t]).to(dev) for t in steps}
        dev_aor = {t: None if aor[t] is None else torch.from_numpy(aor[t]).to(dev) for t in steps}
        # every buffer a pipelined step writes exists before the inputs-ready event
        # (the counters are cleared by the library itself)
        outs = {t: (torch.empty(lab, dtype=torch.int32, device=dev),
                    torch.empty(lab, dtype=torch.uint8, device=dev),
                    torch.empty((lab, width), dtype=torch.float32, device=dev),
                    torch.empty(7, dtype=torch.int64, device=dev)) for t in steps}
        ready = torch.cuda.Event()
        ready.record()
        for t in steps:
            rows, hit, out, st = outs[t]
            binding.mpzch_train_step(tbl.h, dev_ids[t], lab, pool(t)[1], t, rows, hit, out, ao_d,
                                     dev_aor[t], st, inputs_ready=ready)
        torch.cuda.synchronize()
        for t in steps:
            ids = host[t]
            rows_d, hit_d, out_d, st_d = outs[t]
            rc, orows, ohit = orc.lookup(ids[:lab])
            assert rc == 0
            assert_bitwise(rows_d.cpu().numpy(), orows, f"step {t}: rows")
            assert_bitwise(hit_d.cpu().numpy(), ohit, f"step {t}: hit")
            # gathered features: all rows every few steps, a sample otherwise; with a
            # value-row sample only positions whose row is kept (or misses) are checked
            if t % full_gather_every == 0 or t == w.steps - 1:
                pos = np.arange(lab)
            else:
                pos = np.sort(rng.choice(lab, size=min(gather_sample, lab), replace=False))
            if value_rows is not None:
                pos = pos[(ohit[pos] == 0) | tracked[np.maximum(orows[pos], 0)]]
            a = aor[t]
            oout = orc.gather_fused(orows[pos], ohit[pos], ao, None if a is None else a[pos])
            got = out_d[torch.from_numpy(pos).to(dev)].cpu().numpy()
            assert_bitwise(got, oout, f"step {t}: gathered features")
            rc, ost = orc.writeback(ids, pool(t)[0], t)
            assert rc == 0
            gst = stats_dict(st_d)
            for k in STATS_KEYS:
                assert gst[k] == ost[k], (t, k, gst, ost)
        del outs
        t = steps[-1]
        if (t + 1) % check_state_every == 0 or t == w.steps - 1:
            keys, last, _ = tbl.state()
            ok, ol, _ = orc.state()
            assert_bitwise(keys.cpu().numpy(), ok, f"step {t}: keys")
            assert_bitwise(last.cpu().numpy(), ol, f"step {t}: last")
    _, _, M = tbl.state()
    if value_rows is None:
        step = 1 << 20  # rows per compared chunk (2 GiB at 512-d)
        for r0 in range(0, w.capacity, step):
            r1 = min(r0 + step, w.capacity)
            assert_bitwise(M[r0:r1].cpu().numpy(), orc.rows(np.arange(r0, r1, dtype=np.int32)),
                           f"final values rows {r0}..{r1}")
    else:
        idx = torch.from_numpy(value_rows.astype(np.int64)).to(dev)
        assert_bitwise(M.index_select(0, idx).cpu().numpy(), orc.rows(value_rows), "final value rows")
    assert tbl.status() == 0
    return tbl, orc


def test_full_1m_rows_stream():
    tbl, orc = run_full(inputs.CFG2_1M, check_state_every=10, full_gather_every=10)
    tbl.close()


def test_full_multitable_then_export_and_serving():
    from hashed_sparse_table_b200 import binding
    w = inputs.CFG3_MULTI
    tbl, orc = run_full(w, check_state_every=10, full_gather_every=10)
    dev = tbl.device
    # export: rows written in the last 50 steps
    since = w.steps - inputs.CFG5_SERVE_SINCE
    rows_d, cnt_d = tbl.select_written_since(since)
    orows = orc.select_written_since(since)
    n = int(cnt_d.item())
    assert n == orows.size and n > 0
    assert_bitwise(rows_d[:n].cpu().numpy(), orows, "select rows")
    q, s, k = tbl.export_int8(rows_d, n=w.capacity, dev_n=cnt_d)
    oq, os_, ok = orc.export_int8(orows)
    assert_bitwise(q[:n].cpu().numpy(), oq, "int8 q")
    assert_bitwise(s[:n].cpu().numpy(), os_, "scale")
    assert_bitwise(k[:n].cpu().numpy(), ok, "exported keys")
    # serving snapshot (exported rows at their row index) and 4096 x 1024 candidates
    sk, sq, ss = snapshot_from_export(w.capacity, w.dim, orows, oq, os_, ok)
    sk_d, sq_d, ss_d = (torch.from_numpy(x).to(dev) for x in (sk, sq, ss))
    cand = inputs.serve_candidates()
    assert cand.size == inputs.CFG5_REQUESTS * inputs.CFG5_CANDIDATES
    chunk = 512 * inputs.CFG5_CANDIDATES
    out = torch.empty((chunk, w.dim), dtype=torch.float32, device=dev)
    grow = torch.empty(chunk, dtype=torch.int32, device=dev)
    ghit = torch.empty(chunk, dtype=torch.uint8, device=dev)
    hits = 0
    for c0 in range(0, cand.size, chunk):
        ids = cand[c0:c0 + chunk]
        binding.mpzch_serve_gather(sk_d, w.probes, sq_d, ss_d, torch.from_numpy(ids).to(dev),
                                   grow, ghit, out)
        rc, orow, ohit, oout = oracle.serve_gather(sk, w.capacity, w.probes, sq, ss, w.dim, ids)
        assert rc == 0
        assert_bitwise(grow.cpu().numpy(), orow, f"serve rows @{c0}")
        assert_bitwise(ghit.cpu().numpy(), ohit, f"serve hit @{c0}")
        assert_bitwise(out.cpu().numpy(), oout, f"serve features @{c0}")
        hits += int(ohit.sum())
    assert 0 < hits < cand.size
    tbl.close()


def host_available_bytes() -> int:
    with open("/proc/meminfo") as f:
        for line in f:
            if line.startswith("MemAvailable:"):
                return int(line.split()[1]) * 1024
    return 0


def test_full_16m_rows_capacity_stress():
    w = inputs.CFG4_16M
    table_bytes = w.capacity * w.dim * 4
    if host_available_bytes() >= table_bytes + (24 << 30):
        # the oracle keeps every value row: all 32 GiB compared at the end
        value_rows = None
    else:
        value_rows = np.arange(0, w.capacity, 64, dtype=np.int32)
    tbl, orc = run_full(w, check_state_every=20, full_gather_every=25, value_rows=value_rows,
                        chunk=10)
    tbl.close()
