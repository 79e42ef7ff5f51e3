"""mpzch_dedup_static: in-batch dedup without any device allocation.

Some callers cannot call cudaMalloc: a plug-in inside an inference server or
another framework that owns all device memory through its own pool, or a
latency-critical path where an allocation would synchronise the device.  For
them the library offers one dedup entry point whose scratch is a fixed static
device array instead of memory owned by a table handle.  This test calls it
through the C ABI and checks that it returns exactly what the allocating
entry point (mpzch_dedup) returns, on two calls in a row (the second call
sees whatever the first left in the shared array), and that a batch above the
fixed maximum is refused.

The file is named so that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from hashed_sparse_table_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_IDS = 262144  # MPZCH_DEDUP_STATIC_MAX_IDS
ERANGE = -6


def _static_fn():
    from hashed_sparse_table_b200 import binding
    f = binding.lib().mpzch_dedup_static
    p = C.c_void_p
    f.argtypes = [p, C.c_int64, p, p, p, p, p]
    f.restype = C.c_int
    return f


def _ptr(t):
    return C.c_void_p(t.data_ptr())


def test_static_dedup_matches_allocating_dedup_on_two_calls():
    from hashed_sparse_table_b200 import binding
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    f = _static_fn()
    tbl = binding.MpzchTable(1024, 4, 2)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # a large ragged batch, then a smaller one that reuses the same scratch
    for call, (n, alpha, seed) in enumerate([(200_001, 0.9, 11), (70_003, 1.2, 12)]):
        ids = inputs.zipf_keys(np.random.default_rng(seed), alpha, 5_000_000, n)
        ids_d = torch.from_numpy(ids).to(dev)
        want_u, want_p, want_c = tbl.dedup(ids_d)
        uniq = torch.full((n,), -9, dtype=torch.int64, device=dev)
        pos = torch.full((n,), -9, dtype=torch.int32, device=dev)
        cnt = torch.full((1,), -9, dtype=torch.int64, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        rc = f(_ptr(ids_d), n, _ptr(uniq), _ptr(pos), _ptr(cnt), _ptr(status), stream)
        assert rc == 0, (call, rc)
        torch.cuda.synchronize()
        c = int(want_c.item())
        assert int(cnt.item()) == c, call
        # integer outputs: exact equality (tolerance zero, as for every index output)
        assert torch.equal(uniq[:c], want_u[:c]), call
        assert torch.equal(pos[:c], want_p[:c]), call
        assert int(status.item()) == 0
    assert tbl.status() == 0


def test_static_dedup_refuses_batches_above_the_maximum():
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    f = _static_fn()
    ids = torch.zeros(MAX_IDS + 1, dtype=torch.int64, device=dev)
    out = torch.empty(MAX_IDS + 1, dtype=torch.int64, device=dev)
    pos = torch.empty(MAX_IDS + 1, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int64, device=dev)
    rc = f(_ptr(ids), MAX_IDS + 1, _ptr(out), _ptr(pos), _ptr(cnt), None,
           C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ERANGE
