"""Drives one workload through the CUDA library and the CPU oracle side by side
and compares every output bit for bit (GPU tests only)."""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

import oracle
from hashed_sparse_table_b200 import inputs

STATS_KEYS = ("n_ids", "n_unique", "n_hit_unique", "n_inserted", "n_evicted", "n_dropped")


def bits(a: np.ndarray) -> np.ndarray:
    """Bit pattern view: equality on it is byte equality (+0 vs -0, NaN payloads)."""
    a = np.ascontiguousarray(a)
    return a.view({4: np.uint32, 8: np.uint64, 1: np.uint8, 2: np.uint16}[a.dtype.itemsize])


def assert_bitwise(gpu: np.ndarray, ref: np.ndarray, what: str):
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    g, r = bits(gpu), bits(ref)
    if not np.array_equal(g, r):
        bad = np.argwhere(g != r)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: gpu={gpu[i]!r} "
                             f"oracle={ref[i]!r}")


def stats_dict(t: torch.Tensor) -> dict:
    v = t.cpu().tolist()
    return dict(zip(STATS_KEYS + ("n_rounds",), v))


@dataclasses.dataclass
class RunResult:
    tbl: object
    orc: object
    steps: int
    stats: list


def make_pair(w: inputs.Workload, track_all: bool = True, track_rows: Optional[np.ndarray] = None,
              flags: int = 0):
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(w.capacity, w.dim, w.probes, flags=flags)
    orc = oracle.OracleTable(w.capacity, w.dim, w.probes, track_all=track_all)
    if track_rows is not None:
        orc.track_rows(track_rows)
    return tbl, orc


def compare_state(tbl, orc, what: str, value_rows: Optional[np.ndarray] = None, values=True):
    from hashed_sparse_table_b200 import binding
    binding.mpzch_tier_sync(tbl.h)  # an HBM row cache writes its rows back (no-op without one)
    keys, last, M = tbl.state()
    ok, ol, _ = orc.state()
    assert_bitwise(keys.cpu().numpy(), ok, f"{what}: keys")
    assert_bitwise(last.cpu().numpy(), ol, f"{what}: last")
    if not values:
        return
    if value_rows is None:
        assert_bitwise(M.cpu().numpy(), orc.values(), f"{what}: M")
    else:
        idx = torch.from_numpy(value_rows.astype(np.int64)).to(M.device)
        assert_bitwise(M.index_select(0, idx).cpu().numpy(), orc.rows(value_rows), f"{what}: M rows")


def run_pair(w: inputs.Workload, steps: Optional[int] = None, tbl=None, orc=None, start: int = 0,
             state_every: int = 1, values_every: int = 1, value_rows=None, gather_rows: int = -1,
             ids_fn=None, e_fn=None, wide_rounds: Optional[int] = None,
             fused_step: bool = False, eta: Optional[float] = None,
             flags: int = 0, cluster: Optional[int] = None,
             options: Optional[dict] = None) -> RunResult:
    """Runs steps [start, start+steps) of workload w on both sides.

    Per step: lookup of the labeled ids, fused gather (with the always-on concat
    when the workload has one), Writeback of the whole batch.  Compares rows,
    hit, gathered features (first `gather_rows` rows, -1 = all), Writeback
    counters, and the table state every `state_every` / `values_every` steps."""
    from hashed_sparse_table_b200 import binding
    if tbl is None:
        tbl, orc = make_pair(w, flags=flags)
    if wide_rounds is not None:
        binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_WIDE_ROUNDS, wide_rounds)
    if cluster is not None:
        binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_CLUSTER_INSERT, cluster)
    for opt, val in (options or {}).items():
        binding.mpzch_set_option(tbl.h, opt, val)
    if eta is not None:
        binding.mpzch_set_learning_rate(tbl.h, eta)
        orc.set_learning_rate(eta)
    T = w.steps if steps is None else steps
    dev = tbl.device
    ao = inputs.author_table(w)
    ao_d = torch.from_numpy(ao).to(dev) if ao is not None else None
    stats_d = torch.zeros(7, dtype=torch.int64, device=dev)
    all_stats = []
    for t in range(start, start + T):
        ids = ids_fn(t) if ids_fn else inputs.step_ids(w, t)
        e = e_fn(t, ids.size) if e_fn else inputs.step_e(w, t, rows=ids.size)
        lab = min(w.labeled, ids.size)
        ids_d = torch.from_numpy(ids).to(dev)
        e_d = torch.from_numpy(e).to(dev)
        aor = inputs.author_rows(w, ids[:lab])
        aor_d = torch.from_numpy(aor).to(dev) if aor is not None else None
        if fused_step:
            rows_d, hit_d, out_d = tbl.train_step(ids_d, lab, e_d, t, ao_d, aor_d, stats_d)
        else:
            rows_d, hit_d = tbl.lookup(ids_d[:lab])
            out_d = tbl.gather_fused(rows_d, hit_d, ao_d, aor_d)
            tbl.writeback(ids_d, e_d, t, stats_d)
        # oracle
        rc, orows, ohit = orc.lookup(ids[:lab])
        assert rc == 0
        n_g = lab if gather_rows < 0 else min(gather_rows, lab)
        oout = orc.gather_fused(orows[:n_g], ohit[:n_g], ao, None if aor is None else aor[:n_g])
        rc, ost = orc.writeback(ids, e, t)
        assert rc == 0
        assert_bitwise(rows_d.cpu().numpy(), orows, f"step {t}: rows")
        assert_bitwise(hit_d.cpu().numpy(), ohit, f"step {t}: hit")
        assert_bitwise(out_d[:n_g].cpu().numpy(), oout, f"step {t}: gathered features")
        gst = stats_dict(stats_d)
        for k in STATS_KEYS:
            assert gst[k] == ost[k], (t, k, gst, ost)
        assert (gst["n_rounds"] >= 1) == (ost["n_inserted"] > 0), (t, gst)
        all_stats.append(gst)
        last_step = t == start + T - 1
        if last_step or (state_every and (t - start) % state_every == 0):
            with_values = last_step or (values_every and (t - start) % values_every == 0)
            compare_state(tbl, orc, f"step {t}", value_rows, values=with_values)
    assert tbl.status() == 0
    return RunResult(tbl, orc, T, all_stats)


def snapshot_from_export(capacity: int, dim: int, rows: np.ndarray, q: np.ndarray, scale: np.ndarray,
                         keys: np.ndarray):
    """Serving snapshot image: exported rows at their own row index, -1 elsewhere."""
    snap_keys = np.full(capacity, -1, np.int64)
    snap_q = np.zeros((capacity, dim), np.int8)
    snap_s = np.zeros(capacity, np.float32)
    snap_keys[rows] = keys
    snap_q[rows] = q
    snap_s[rows] = scale
    return snap_keys, snap_q, snap_s


def run_pipelined(w: inputs.Workload, steps: Optional[int] = None, flags: int = 0,
                  cluster: Optional[int] = None, options: Optional[dict] = None):
    """All steps' inputs uploaded first, then every step issued back to back as
    a pipelined mpzch_train_step (inputs_ready = one event after the uploads),
    each step with its own output buffers; then every output and the final
    table are compared with the oracle run step by step.  The table is not
    reserved, so the first step grows the per-batch scratch after the event was
    recorded (the growth must complete before the helper streams use it)."""
    from hashed_sparse_table_b200 import binding
    T = w.steps if steps is None else steps
    tbl, orc = make_pair(w, flags=flags)
    if cluster is not None:
        binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_CLUSTER_INSERT, cluster)
    for opt, val in (options or {}).items():
        binding.mpzch_set_option(tbl.h, opt, val)
    dev = tbl.device
    ao = inputs.author_table(w)
    ao_d = torch.from_numpy(ao).to(dev) if ao is not None else None
    host = []
    for t in range(T):
        ids = inputs.step_ids(w, t)
        e = inputs.step_e(w, t, rows=ids.size)
        host.append((ids, e, inputs.author_rows(w, ids[:w.labeled])))
    dev_in = [(torch.from_numpy(i).to(dev), torch.from_numpy(e).to(dev),
               None if a is None else torch.from_numpy(a).to(dev)) for i, e, a in host]
    lab = w.labeled
    width = w.dim + (0 if ao is None else ao.shape[1])
    # every buffer a pipelined step writes exists before the inputs-ready event
    # (the counters are cleared by the library itself)
    outs = [(torch.empty(lab, dtype=torch.int32, device=dev),
             torch.empty(lab, dtype=torch.uint8, device=dev),
             torch.empty((lab, width), dtype=torch.float32, device=dev),
             torch.empty(7, dtype=torch.int64, device=dev)) for _ in range(T)]
    ready = torch.cuda.Event()
    ready.record()
    for t in range(T):
        ids_d, e_d, aor_d = dev_in[t]
        rows, hit, out, st = outs[t]
        binding.mpzch_train_step(tbl.h, ids_d, lab, e_d, t, rows, hit, out, ao_d, aor_d, st,
                                 inputs_ready=ready)
    torch.cuda.synchronize()
    for t in range(T):
        ids, e, aor = host[t]
        rows, hit, out, st = outs[t]
        rc, orows, ohit = orc.lookup(ids[:lab])
        oout = orc.gather_fused(orows, ohit, ao, aor)
        rc, ost = orc.writeback(ids, e, t)
        assert_bitwise(rows.cpu().numpy(), orows, f"pipelined step {t}: rows")
        assert_bitwise(hit.cpu().numpy(), ohit, f"pipelined step {t}: hit")
        assert_bitwise(out.cpu().numpy(), oout, f"pipelined step {t}: features")
        gst = stats_dict(st)
        for k in STATS_KEYS:
            assert gst[k] == ost[k], (t, k, gst, ost)
    compare_state(tbl, orc, "after pipelined steps")
    assert tbl.status() == 0
    return tbl, orc
