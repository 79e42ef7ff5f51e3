"""Streaming export to a host serving snapshot (RES) against the oracle.

Training steps stream the rows written since the previous export every few
steps; after a flush, the published snapshot must equal, row by row and bit for
bit, the oracle's table at that step: live keys, last-write steps, and the
int8 export (q, scale) of every live row; rows never written stay empty.
The serving gather then reads the streamed snapshot.
"""
import numpy as np
import pytest
import torch

import oracle
from hashed_sparse_table_b200 import inputs
from gpu_harness import assert_bitwise, make_pair

pytestmark = pytest.mark.gpu

W = inputs.Workload("res_c3_small", 3, capacity=1 << 13, dim=128, probes=8, steps=24,
                    labeled=700, pool=2900, zipf_alpha=0.9, zipf_keys=40_000,
                    ao_rows=1 << 13, ao_dim=16, ao_kind="mix")


def oracle_snapshot(orc):
    keys, last, _ = orc.state()
    live = np.nonzero(keys >= 0)[0].astype(np.int32)
    q, s, k = orc.export_int8(live)
    snap_q = np.zeros((orc.capacity, orc.dim), np.int8)
    snap_s = np.zeros(orc.capacity, np.float32)
    snap_q[live] = q
    snap_s[live] = s
    return keys, last, snap_q, snap_s


def check_snapshot(res, orc, upto, what):
    keys, q, scale, last, version, got_upto = res.read()
    okeys, olast, oq, os_ = oracle_snapshot(orc)
    assert got_upto == upto, what
    assert_bitwise(keys, okeys, f"{what}: keys")
    assert_bitwise(last, olast, f"{what}: last")
    assert_bitwise(scale, os_, f"{what}: scale")
    assert_bitwise(q, oq, f"{what}: int8 rows")
    return version


@pytest.mark.parametrize("pipelined", [False, True])
def test_streamed_snapshot_equals_oracle_table(pipelined):
    from hashed_sparse_table_b200 import binding
    tbl, orc = make_pair(W)
    res = binding.MpzchRes(tbl, slots=2, period_ms=50)
    dev = tbl.device
    ao = inputs.author_table(W)
    ao_d = torch.from_numpy(ao).to(dev)
    lab = W.labeled
    streamed_upto = -1
    versions = []
    for t in range(W.steps):
        ids = inputs.step_ids(W, t)
        e = inputs.step_e(W, t)
        aor = inputs.author_rows(W, ids[:lab])
        ids_d, e_d, aor_d = (torch.from_numpy(x).to(dev) for x in (ids, e, aor))
        rows = torch.empty(lab, dtype=torch.int32, device=dev)
        hit = torch.empty(lab, dtype=torch.uint8, device=dev)
        out = torch.empty((lab, W.dim + W.ao_dim), dtype=torch.float32, device=dev)
        st = torch.empty(7, dtype=torch.int64, device=dev)
        ready = None
        if pipelined:
            ready = torch.cuda.Event()
            ready.record()
        binding.mpzch_train_step(tbl.h, ids_d, lab, e_d, t, rows, hit, out, ao_d, aor_d, st,
                                 inputs_ready=ready)
        orc.writeback(ids, e, t)
        if t % 3 == 2:
            rc = res.stream(streamed_upto + 1, t)
            if rc == binding.MPZCH_OK:
                streamed_upto = t
        if t in (11, W.steps - 1):
            if streamed_upto < t:  # the last export was skipped or is older: stream the rest
                while res.stream(streamed_upto + 1, t) == binding.MPZCH_EBUSY:
                    res.flush()
                streamed_upto = t
            res.flush()
            versions.append(check_snapshot(res, orc, t, f"after step {t}"))
    assert versions[1] > versions[0] >= 1
    lat = res.latency()
    assert lat["samples"] >= 2 and lat["overflow_rows"] == 0
    assert 0 <= lat["p50_ms"] <= lat["p99_ms"] <= lat["max_ms"]
    # serving from the streamed snapshot equals serving from the oracle's export
    keys, q, scale, last, _, _ = res.read()
    okeys, _, oq, os_ = oracle_snapshot(orc)
    cand = inputs.zipf_keys(np.random.default_rng(7), 0.9, W.zipf_keys, 4000)
    rc, orow, ohit, oout = oracle.serve_gather(okeys, W.capacity, W.probes, oq, os_, W.dim, cand)
    assert rc == 0
    out = torch.empty((cand.size, W.dim), dtype=torch.float32, device=dev)
    grow = torch.empty(cand.size, dtype=torch.int32, device=dev)
    ghit = torch.empty(cand.size, dtype=torch.uint8, device=dev)
    binding.mpzch_serve_gather(torch.from_numpy(keys).to(dev), W.probes,
                               torch.from_numpy(q).to(dev), torch.from_numpy(scale).to(dev),
                               torch.from_numpy(cand).to(dev), grow, ghit, out)
    assert_bitwise(grow.cpu().numpy(), orow, "serve rows from the streamed snapshot")
    assert_bitwise(out.cpu().numpy(), oout, "serve features from the streamed snapshot")
    res.close()
    assert tbl.status() == 0


def test_busy_slots_are_reported_and_covered_later():
    from hashed_sparse_table_b200 import binding
    tbl, orc = make_pair(W)
    res = binding.MpzchRes(tbl, slots=1, period_ms=10_000)
    dev = tbl.device
    codes = []
    for t in range(6):
        ids = inputs.step_ids(W, t)
        e = inputs.step_e(W, t)
        tbl.writeback(torch.from_numpy(ids).to(dev), torch.from_numpy(e).to(dev), t)
        orc.writeback(ids, e, t)
        codes.append(res.stream(0, t))  # always everything since step 0
    assert codes[0] == binding.MPZCH_OK
    assert set(codes) <= {binding.MPZCH_OK, binding.MPZCH_EBUSY}
    while res.stream(0, 5) == binding.MPZCH_EBUSY:
        res.flush()
    res.flush()
    check_snapshot(res, orc, 5, "after busy slots")
    res.close()


def test_max_rows_overflow_is_counted():
    from hashed_sparse_table_b200 import binding
    tbl, orc = make_pair(W)
    res = binding.MpzchRes(tbl, max_rows=100, slots=1, period_ms=10)
    ids = inputs.step_ids(W, 0)
    e = inputs.step_e(W, 0)
    tbl.writeback(torch.from_numpy(ids).cuda(), torch.from_numpy(e).cuda(), 0)
    orc.writeback(ids, e, 0)
    assert res.stream(0, 0) == binding.MPZCH_OK
    res.flush()
    lat = res.latency()
    n_written = int((orc.state()[0] >= 0).sum())
    assert lat["overflow_rows"] == n_written - 100
    keys, _, _, _, _, _ = res.read()
    assert (keys >= 0).sum() == 100
    res.close()
