"""Hot/cold value tier (values in host memory + an HBM cache of rows) vs the
CPU oracle, bit for bit.

The cache must be invisible: gathered features every step, Writeback
counters, and -- after writing the cache back -- every value row equal to the
oracle's, for caches from one slot to the whole table, with separate calls,
the fused step and pipelined steps; the int8 export (which writes the cache
back by itself); a restore of the host values followed by a discard of the
cache; and the option's argument checks.
"""
import numpy as np
import pytest
import torch

import oracle
from hashed_sparse_table_b200 import inputs
from gpu_harness import assert_bitwise, compare_state, make_pair, run_pair, run_pipelined
from test_gpu_parity import SCALED

pytestmark = pytest.mark.gpu


def _tier(rows):
    from hashed_sparse_table_b200 import binding
    return {binding.MPZCH_OPT_HBM_CACHE_ROWS: rows}


def _host():
    from hashed_sparse_table_b200 import binding
    return binding.MPZCH_VALUES_IN_HOST_MEMORY


@pytest.mark.parametrize("name,rows", [("c3_small", 2048), ("c2_small", 4096), ("c4_stress", 1024),
                                       ("nonpow2", 512), ("c3_small", 1), ("c3_small", 8192)])
@pytest.mark.parametrize("fused", [False, True])
def test_tier_bit_exact_every_step(name, rows, fused):
    run_pair(SCALED[name], fused_step=fused, flags=_host(), options=_tier(rows))


@pytest.mark.parametrize("name", ["c3_small", "c4_stress"])
def test_tier_pipelined_steps_bit_exact(name):
    run_pipelined(SCALED[name], flags=_host(), options=_tier(1024))


def test_tier_learning_rate_and_resize_mid_stream():
    """A general learning rate, and the cache resized (written back, rebuilt)
    between steps: still the values of one plain table."""
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"].scaled(steps=6)
    r = run_pair(w, eta=0.5, flags=_host(), options=_tier(512))
    binding.mpzch_set_option(r.tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS, 4096)
    run_pair(w, tbl=r.tbl, orc=r.orc, start=w.steps, steps=4)
    binding.mpzch_set_option(r.tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS, 0)
    run_pair(w, tbl=r.tbl, orc=r.orc, start=w.steps + 4, steps=3)


def test_tier_export_writes_the_cache_back():
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"].scaled(steps=8)
    r = run_pair(w, flags=_host(), options=_tier(2048), state_every=0)
    tbl, orc = r.tbl, r.orc
    rows_d, cnt = tbl.select_written_since(3)
    n = int(cnt.item())
    orows = orc.select_written_since(3)
    assert_bitwise(rows_d[:n].cpu().numpy(), orows, "select")
    q, s, k = tbl.export_int8(rows_d, n=w.capacity, dev_n=cnt)
    oq, os_, ok = orc.export_int8(orows)
    assert_bitwise(q[:n].cpu().numpy(), oq, "int8 q")
    assert_bitwise(s[:n].cpu().numpy(), os_, "scale")
    assert_bitwise(k[:n].cpu().numpy(), ok, "keys")


def test_tier_restore_then_discard():
    """Host values replaced by the caller (a restore): discarding the cache
    makes the table read the restored values."""
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"].scaled(steps=5)
    r = run_pair(w, flags=_host(), options=_tier(2048))
    tbl, orc = r.tbl, r.orc
    _, _, M = tbl.state()
    rng = np.random.default_rng(8)
    vals = rng.standard_normal((w.capacity, w.dim)).astype(np.float32)
    M.copy_(torch.from_numpy(vals))
    binding.mpzch_tier_sync(tbl.h, discard=True)
    for row in range(w.capacity):
        orc.set_row(row, vals[row])
    run_pair(w, tbl=tbl, orc=orc, start=w.steps, steps=3)


def test_tier_option_checks():
    from hashed_sparse_table_b200 import binding
    dev_tbl = binding.MpzchTable(1024, 8, 4)
    with pytest.raises(binding.MpzchError):  # values in device memory
        binding.mpzch_set_option(dev_tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS, 256)
    tbl = binding.MpzchTable(1024, 8, 4, flags=_host())
    for bad in (3, 2048, -1):
        with pytest.raises(binding.MpzchError):
            binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS, bad)
    binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS, 256)
    assert binding.mpzch_get_option(tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS) == 256
    binding.mpzch_tier_sync(dev_tbl.h)  # no cache: no-op


@pytest.mark.parametrize("rows", [1, 512, 1 << 13])
def test_tier_counters_account_for_every_row(rows):
    """The tier counters against the oracle's step counters and lookups: every
    written row's e_hat is read once (cache or host) and its result written
    once, every gathered hit is read once, and a row is read from the cache
    only after it was written there.  With a cache of the whole table (one
    slot per row) no result goes to the host, nothing is written back, every
    gathered hit comes from the cache, and a row's e_hat comes from the host
    exactly once (its first write), so host reads = rows holding a key at the
    end.  Reset zeroes the counters."""
    from hashed_sparse_table_b200 import binding
    w = SCALED["c3_small"].scaled(steps=10)
    tbl, orc = make_pair(w, flags=_host())
    binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_HBM_CACHE_ROWS, rows)
    dev = tbl.device
    ao = inputs.author_table(w)
    ao_d = torch.from_numpy(ao).to(dev)
    stats_d = torch.zeros(7, dtype=torch.int64, device=dev)
    written = hits = 0
    for t in range(w.steps):
        ids = inputs.step_ids(w, t)
        e = inputs.step_e(w, t, rows=ids.size)
        lab = min(w.labeled, ids.size)
        aor = inputs.author_rows(w, ids[:lab])
        tbl.train_step(torch.from_numpy(ids).to(dev), lab, torch.from_numpy(e).to(dev), t, ao_d,
                       torch.from_numpy(aor).to(dev), stats_d)
        rc, _, ohit = orc.lookup(ids[:lab])
        assert rc == 0
        hits += int(ohit.sum())
        rc, ost = orc.writeback(ids, e, t)
        assert rc == 0
        written += ost["n_unique"] - ost["n_dropped"]
    st = binding.mpzch_tier_stats(tbl.h)
    assert st["update_read_cache"] + st["update_read_host"] == written, st
    assert st["update_write_cache"] + st["update_write_host"] == written, st
    assert st["gather_cache"] + st["gather_host"] == hits, st
    assert st["update_read_cache"] <= st["update_write_cache"], st
    if rows == w.capacity:
        keys, _, _ = orc.state()
        assert st["update_write_host"] == 0 and st["write_back"] == 0, st
        assert st["gather_host"] == 0, st
        assert st["update_read_host"] == int((keys != -1).sum()), st
    elif rows > 1:
        assert st["write_back"] > 0 and st["update_read_cache"] > 0, st
    st2 = binding.mpzch_tier_stats(tbl.h, reset=True)
    assert st2 == st
    assert set(binding.mpzch_tier_stats(tbl.h).values()) == {0}
    assert tbl.status() == 0
