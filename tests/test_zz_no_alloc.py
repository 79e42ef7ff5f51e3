"""mpzch_dedup_static: in-batch dedup without any device allocation.

Some callers cannot call cudaMalloc: a plug-in inside an inference server or
another framework that owns all device memory through its own pool, or a
latency-critical path where an allocation would synchronise the device.  For
them the library offers one dedup entry point whose scratch is a fixed static
device array instead of memory owned by a table handle.  These tests call it
through the C ABI and check that it returns exactly what the allocating entry
point (mpzch_dedup) returns and what the CPU oracle's dedup returns, on two
calls in a row (the second call sees whatever the first left in the shared
array); that negative ids are skipped and flagged as mpzch_dedup does; that an
empty batch gives a zero count; that a NULL status pointer is accepted; and
that a batch above the fixed maximum is refused.

The file is named so that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from hashed_sparse_table_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_IDS = 262144  # MPZCH_DEDUP_STATIC_MAX_IDS
ERANGE = -6
STATUS_BADKEY = 1


def _static_fn():
    from hashed_sparse_table_b200 import binding
    f = binding.lib().mpzch_dedup_static
    p = C.c_void_p
    f.argtypes = [p, C.c_int64, p, p, p, p, p]
    f.restype = C.c_int
    return f


def _ptr(t):
    return C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _static_dedup(f, ids_d, with_status=True):
    n = ids_d.numel()
    dev = ids_d.device
    uniq = torch.full((max(n, 1),), -9, dtype=torch.int64, device=dev)
    pos = torch.full((max(n, 1),), -9, dtype=torch.int32, device=dev)
    cnt = torch.full((1,), -9, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = f(_ptr(ids_d) if n else None, n, _ptr(uniq) if n else None, _ptr(pos) if n else None,
           _ptr(cnt), _ptr(status) if with_status else None, _stream())
    assert rc == 0, rc
    torch.cuda.synchronize()
    c = int(cnt.item())
    return uniq[:c].cpu().numpy(), pos[:c].cpu().numpy(), c, int(status.item())


def test_static_dedup_matches_allocating_dedup_and_oracle_on_two_calls():
    from hashed_sparse_table_b200 import binding
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    f = _static_fn()
    tbl = binding.MpzchTable(1024, 4, 2)
    # a large ragged batch, then a smaller one that reuses the same scratch
    for call, (n, alpha, seed) in enumerate([(200_001, 0.9, 11), (70_003, 1.2, 12)]):
        ids = inputs.zipf_keys(np.random.default_rng(seed), alpha, 5_000_000, n)
        ids_d = torch.from_numpy(ids).to(dev)
        want_u, want_p, want_c = tbl.dedup(ids_d)
        u, p, c, st = _static_dedup(f, ids_d)
        wc = int(want_c.item())
        # integer outputs: exact equality (tolerance zero, as for every index output)
        assert c == wc, call
        assert np.array_equal(u, want_u[:wc].cpu().numpy()), call
        assert np.array_equal(p, want_p[:wc].cpu().numpy()), call
        assert st == 0
        ou, op = oracle.dedup(ids)
        assert np.array_equal(u, ou), call
        assert np.array_equal(p.astype(np.int64), op), call
    assert tbl.status() == 0


def test_static_dedup_negative_ids_empty_batch_and_null_status():
    from hashed_sparse_table_b200 import binding
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    f = _static_fn()
    tbl = binding.MpzchTable(1024, 4, 2)
    rng = np.random.default_rng(5)
    ids = inputs.zipf_keys(rng, 1.05, 10_000, 3_001)
    bad = rng.choice(ids.size, 17, replace=False)
    ids[bad] = -1 - rng.integers(0, 1 << 40, bad.size)
    ids_d = torch.from_numpy(ids).to(dev)
    u, p, c, st = _static_dedup(f, ids_d)
    assert st & STATUS_BADKEY
    want_u, want_p, want_c = tbl.dedup(ids_d)
    wc = int(want_c.item())
    assert c == wc
    assert np.array_equal(u, want_u[:wc].cpu().numpy())
    assert np.array_equal(p, want_p[:wc].cpu().numpy())
    assert tbl.status() & STATUS_BADKEY
    ou, op = oracle.dedup(ids)
    assert np.array_equal(u, ou) and np.array_equal(p.astype(np.int64), op)
    # empty batch: count 0, nothing launched that reads ids
    u0, p0, c0, st0 = _static_dedup(f, torch.empty(0, dtype=torch.int64, device=dev))
    assert c0 == 0 and st0 == 0
    # a launching call without a status word
    good = torch.from_numpy(np.abs(ids)).to(dev)
    u1, p1, c1, _ = _static_dedup(f, good, with_status=False)
    ou1, op1 = oracle.dedup(np.abs(ids))
    assert c1 == ou1.size
    assert np.array_equal(u1, ou1) and np.array_equal(p1.astype(np.int64), op1)


def test_static_dedup_refuses_batches_above_the_maximum():
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    f = _static_fn()
    ids = torch.zeros(MAX_IDS + 1, dtype=torch.int64, device=dev)
    out = torch.empty(MAX_IDS + 1, dtype=torch.int64, device=dev)
    pos = torch.empty(MAX_IDS + 1, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int64, device=dev)
    rc = f(_ptr(ids), MAX_IDS + 1, _ptr(out), _ptr(pos), _ptr(cnt), None, _stream())
    assert rc == ERANGE
