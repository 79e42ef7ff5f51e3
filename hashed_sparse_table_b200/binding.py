"""Thin ctypes binding of libmpzch.so (argument marshalling only).

Every function here has the name of the C entry point it calls (see
``include/mpzch.h``), takes torch CUDA tensors where the C call takes device
pointers, passes the current CUDA stream unless one is given, and raises
``MpzchError`` on a negative return code.  All table work runs in the CUDA
kernels of the library; there is no other implementation behind this module.
If the built library is missing, importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmpzch.so")

MPZCH_OK = 0
MPZCH_EINVAL = -1
MPZCH_ENOMEM = -2
MPZCH_ECUDA = -3
MPZCH_ECAPTURE = -5
MPZCH_ERANGE = -6
MPZCH_EBUSY = -7
MPZCH_ETIMEDOUT = -8
MPZCH_STATUS_BADKEY = 1
MPZCH_STATUS_BADROW = 2
MPZCH_STATUS_BADAO = 4
MPZCH_STATUS_INTERNAL = 8
MPZCH_STATUS_TIMEOUT = 16
MPZCH_NPHASES = 7
MPZCH_OPT_WIDE_ROUNDS = 1
MPZCH_VALUES_IN_HOST_MEMORY = 1
MPZCH_OPT_SIDE_PRIORITY = 2
MPZCH_OPT_ROW_GRID = 3
MPZCH_OPT_CLUSTER_INSERT = 4
MPZCH_OPT_ROW_KERNEL = 5
MPZCH_OPT_BULK_WARPS = 6
MPZCH_OPT_BULK_BLOCKS = 7
MPZCH_OPT_L2_HINT_ROWS = 8
MPZCH_OPT_WRITE_LIST = 9
MPZCH_OPT_HBM_CACHE_ROWS = 10
PHASES = ("lookup", "gather", "dedup", "insert", "writeback", "select", "export")
STATS_FIELDS = ("n_ids", "n_unique", "n_hit_unique", "n_inserted", "n_evicted", "n_dropped",
                "n_rounds")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmpzch.so is not built ({LIB_PATH}); run "
                      "`python -m hashed_sparse_table_b200.build`")

_lib = C.CDLL(LIB_PATH)
_p, _i64, _i32 = C.c_void_p, C.c_int64, C.c_int32
_SIGS = {
    "mpzch_create": [_i64, _i32, _i32, _p, C.POINTER(_p)],
    "mpzch_create_ex": [_i64, _i32, _i32, C.c_uint32, _p, C.POINTER(_p)],
    "mpzch_destroy": [_p],
    "mpzch_reserve": [_p, _i64, _p],
    "mpzch_lookup": [_p, _p, _i64, _p, _p, _p],
    "mpzch_gather_fused": [_p, _p, _p, _i64, _p, _i64, _i32, _p, _p, _p],
    "mpzch_dedup": [_p, _p, _i64, _p, _p, _p, _p],
    "mpzch_writeback": [_p, _p, _p, _i64, _i64, _p, _p],
    "mpzch_train_step": [_p, _p, _i64, _i64, _p, _i64, _p, _i64, _i32, _p, _p, _p, _p, _p, _p,
                         _p],
    "mpzch_select_written_since": [_p, _i64, _p, _p, _p],
    "mpzch_export_int8": [_p, _p, _i64, _p, _p, _p, _p, _p],
    "mpzch_serve_gather": [_p, _i64, _i32, _p, _p, _i32, _p, _i64, _p, _p, _p, _p, _p],
    "mpzch_state_views": [_p, C.POINTER(_p), C.POINTER(_p), C.POINTER(_p)],
    "mpzch_get_last_step": [_p, C.POINTER(_i64)],
    "mpzch_set_last_step": [_p, _i64],
    "mpzch_get_status": [_p, C.POINTER(_i32), _p],
    "mpzch_trace_enable": [_p, _i32],
    "mpzch_trace_read": [_p, C.POINTER(C.c_double), C.POINTER(_i64), _i32],
    "mpzch_set_option": [_p, _i32, _i64],
    "mpzch_get_option": [_p, _i32, C.POINTER(_i64)],
    "mpzch_tier_sync": [_p, _i32, _p],
    "mpzch_tier_stats": [_p, _p, _i32, _p],
    "mpzch_debug_fail_allocs": [_i32],
    "mpzch_set_learning_rate": [_p, C.c_float],
    "mpzch_res_create": [_p, _i64, _i32, _i32, C.POINTER(_p)],
    "mpzch_res_stream": [_p, _i64, _i64, _p],
    "mpzch_res_flush": [_p, _i32],
    "mpzch_res_read": [_p, _p, _p, _p, _p, C.POINTER(_i64), C.POINTER(_i64)],
    "mpzch_res_latency": [_p, C.POINTER(C.c_double), C.POINTER(C.c_double),
                          C.POINTER(C.c_double), C.POINTER(_i64), C.POINTER(_i64)],
    "mpzch_res_destroy": [_p],
    "mpzch_owner_partition": [_p, _p, _i64, _p, _i32, _p, _i32, _p, _p, _p, _p, _p, _i64, _p],
    "mpzch_owner_combine": [_p, _p, _i64, _i32, _i64, _p, _p, _i32, _p, _i64, _i32, _p, _p, _p,
                            _p, _p, _p],
}
for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = C.c_int
_lib.mpzch_launch_count.argtypes = []
_lib.mpzch_launch_count.restype = _i64
_lib.mpzch_owner_partition_workspace.argtypes = [_i64, _i32]
_lib.mpzch_owner_partition_workspace.restype = _i64
MPZCH_MAX_OWNERS = 256


class MpzchError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed with code {code}")
        self.code = code


def _check(fn: str, rc: int) -> None:
    if rc != MPZCH_OK:
        raise MpzchError(fn, rc)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _need(t: torch.Tensor, dtype, name: str):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got "
                         f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")


def lib() -> C.CDLL:
    return _lib


# ------------------------------------------------------------------ entry points
def mpzch_create(capacity: int, dim: int, probes: int, stream=None) -> C.c_void_p:
    h = C.c_void_p()
    _check("mpzch_create", _lib.mpzch_create(capacity, dim, probes, _stream(stream), C.byref(h)))
    return h


def mpzch_create_ex(capacity: int, dim: int, probes: int, flags: int, stream=None) -> C.c_void_p:
    h = C.c_void_p()
    _check("mpzch_create_ex", _lib.mpzch_create_ex(capacity, dim, probes, flags, _stream(stream),
                                                   C.byref(h)))
    return h


def mpzch_destroy(h) -> None:
    _check("mpzch_destroy", _lib.mpzch_destroy(h))


def mpzch_reserve(h, max_batch: int, stream=None) -> None:
    _check("mpzch_reserve", _lib.mpzch_reserve(h, max_batch, _stream(stream)))


def mpzch_lookup(h, ids, rows, hit, stream=None) -> None:
    _need(ids, torch.int64, "ids")
    _need(rows, torch.int32, "rows")
    _need(hit, torch.uint8, "hit")
    n = ids.numel()
    assert rows.numel() >= n and hit.numel() >= n
    _check("mpzch_lookup", _lib.mpzch_lookup(h, _ptr(ids), n, _ptr(rows), _ptr(hit), _stream(stream)))


def mpzch_gather_fused(h, rows, hit, out, ao_table=None, ao_rows=None, stream=None, n=None) -> None:
    n = rows.numel() if n is None else n
    _need(rows, torch.int32, "rows")
    _need(hit, torch.uint8, "hit")
    _need(out, torch.float32, "out")
    ao_n, ao_dim = 0, 0
    if ao_table is not None:
        _need(ao_table, torch.float32, "ao_table")
        _need(ao_rows, torch.int32, "ao_rows")
        ao_n, ao_dim = ao_table.shape
    _check("mpzch_gather_fused", _lib.mpzch_gather_fused(
        h, _ptr(rows), _ptr(hit), n, _ptr(ao_table), ao_n, ao_dim, _ptr(ao_rows), _ptr(out),
        _stream(stream)))


def mpzch_dedup(h, ids, uniq, pos, count, stream=None) -> None:
    _need(ids, torch.int64, "ids")
    _need(uniq, torch.int64, "uniq")
    _need(pos, torch.int32, "pos")
    _need(count, torch.int64, "count")
    _check("mpzch_dedup", _lib.mpzch_dedup(h, _ptr(ids), ids.numel(), _ptr(uniq), _ptr(pos),
                                           _ptr(count), _stream(stream)))


def mpzch_writeback(h, ids, e, step: int, stats=None, stream=None) -> None:
    _need(ids, torch.int64, "ids")
    _need(e, torch.float32, "e")
    if stats is not None:
        _need(stats, torch.int64, "stats")
        assert stats.numel() >= 7
    n = ids.numel()
    assert e.dim() == 2 and e.shape[0] >= n
    _check("mpzch_writeback", _lib.mpzch_writeback(h, _ptr(ids), _ptr(e), n, step, _ptr(stats),
                                                   _stream(stream)))


def mpzch_train_step(h, ids, n_labeled: int, e, step: int, rows, hit, out, ao_table=None,
                     ao_rows=None, stats=None, inputs_ready=None, stream=None) -> None:
    """inputs_ready: None or a torch.cuda.Event recorded after this step's inputs."""
    _need(ids, torch.int64, "ids")
    _need(e, torch.float32, "e")
    n = ids.numel()
    assert 0 <= n_labeled <= n and e.dim() == 2 and e.shape[0] >= n
    if n_labeled:
        _need(rows, torch.int32, "rows")
        _need(hit, torch.uint8, "hit")
        _need(out, torch.float32, "out")
    ao_n, ao_dim = 0, 0
    if ao_table is not None:
        _need(ao_table, torch.float32, "ao_table")
        _need(ao_rows, torch.int32, "ao_rows")
        ao_n, ao_dim = ao_table.shape
    if stats is not None:
        _need(stats, torch.int64, "stats")
        assert stats.numel() >= 7
    _check("mpzch_train_step", _lib.mpzch_train_step(
        h, _ptr(ids), n, n_labeled, _ptr(e), step, _ptr(ao_table), ao_n, ao_dim, _ptr(ao_rows),
        _ptr(rows), _ptr(hit), _ptr(out), _ptr(stats),
        None if inputs_ready is None else C.c_void_p(inputs_ready.cuda_event), _stream(stream)))


def mpzch_select_written_since(h, since: int, rows_out, count, stream=None) -> None:
    _need(rows_out, torch.int32, "rows_out")
    _need(count, torch.int64, "count")
    _check("mpzch_select_written_since", _lib.mpzch_select_written_since(
        h, since, _ptr(rows_out), _ptr(count), _stream(stream)))


def mpzch_export_int8(h, rows, q, scale, keys_out, n=None, dev_n=None, stream=None) -> None:
    _need(rows, torch.int32, "rows")
    _need(q, torch.int8, "q")
    _need(scale, torch.float32, "scale")
    _need(keys_out, torch.int64, "keys_out")
    if dev_n is not None:
        _need(dev_n, torch.int64, "dev_n")
    n = rows.numel() if n is None else n
    _check("mpzch_export_int8", _lib.mpzch_export_int8(
        h, _ptr(rows), n, _ptr(dev_n), _ptr(q), _ptr(scale), _ptr(keys_out), _stream(stream)))


def mpzch_serve_gather(snap_keys, probes: int, snap_q, snap_scale, ids, rows, hit, out,
                       status=None, stream=None) -> None:
    _need(snap_keys, torch.int64, "snap_keys")
    _need(snap_q, torch.int8, "snap_q")
    _need(snap_scale, torch.float32, "snap_scale")
    _need(ids, torch.int64, "ids")
    _need(rows, torch.int32, "rows")
    _need(hit, torch.uint8, "hit")
    _need(out, torch.float32, "out")
    if status is not None:
        _need(status, torch.int32, "status")
    cap, dim = snap_q.shape
    _check("mpzch_serve_gather", _lib.mpzch_serve_gather(
        _ptr(snap_keys), cap, probes, _ptr(snap_q), _ptr(snap_scale), dim, _ptr(ids), ids.numel(),
        _ptr(rows), _ptr(hit), _ptr(out), _ptr(status), _stream(stream)))


def mpzch_state_views(h):
    k, l, m = C.c_void_p(), C.c_void_p(), C.c_void_p()
    _check("mpzch_state_views", _lib.mpzch_state_views(h, C.byref(k), C.byref(l), C.byref(m)))
    return k.value, l.value, m.value


def mpzch_get_last_step(h) -> int:
    s = C.c_int64()
    _check("mpzch_get_last_step", _lib.mpzch_get_last_step(h, C.byref(s)))
    return s.value


def mpzch_set_last_step(h, step: int) -> None:
    _check("mpzch_set_last_step", _lib.mpzch_set_last_step(h, step))


def mpzch_get_status(h, stream=None) -> int:
    s = C.c_int32()
    _check("mpzch_get_status", _lib.mpzch_get_status(h, C.byref(s), _stream(stream)))
    return s.value


def mpzch_trace_enable(h, on: bool) -> None:
    _check("mpzch_trace_enable", _lib.mpzch_trace_enable(h, 1 if on else 0))


def mpzch_trace_read(h):
    ms = (C.c_double * MPZCH_NPHASES)()
    ln = (C.c_int64 * MPZCH_NPHASES)()
    _check("mpzch_trace_read", _lib.mpzch_trace_read(h, ms, ln, MPZCH_NPHASES))
    return {p: (ms[i], ln[i]) for i, p in enumerate(PHASES)}


def mpzch_set_option(h, option: int, value: int) -> None:
    _check("mpzch_set_option", _lib.mpzch_set_option(h, option, value))


def mpzch_get_option(h, option: int) -> int:
    v = _i64(0)
    _check("mpzch_get_option", _lib.mpzch_get_option(h, option, C.byref(v)))
    return int(v.value)


def mpzch_tier_sync(h, discard: bool = False, stream=None) -> None:
    _check("mpzch_tier_sync", _lib.mpzch_tier_sync(h, 1 if discard else 0, _stream(stream)))


TIER_STAT_NAMES = ("update_read_cache", "update_read_host", "update_write_cache",
                   "update_write_host", "write_back", "gather_cache", "gather_host")


def mpzch_tier_stats(h, reset: bool = False, stream=None) -> dict:
    """Hot/cold tier counters (see include/mpzch.h), as a dict of ints."""
    out = (C.c_int64 * len(TIER_STAT_NAMES))()
    _check("mpzch_tier_stats", _lib.mpzch_tier_stats(h, out, 1 if reset else 0, _stream(stream)))
    return dict(zip(TIER_STAT_NAMES, (int(x) for x in out)))


def mpzch_set_learning_rate(h, eta: float) -> None:
    _check("mpzch_set_learning_rate", _lib.mpzch_set_learning_rate(h, float(eta)))


def mpzch_debug_fail_allocs(count: int) -> None:
    _check("mpzch_debug_fail_allocs", _lib.mpzch_debug_fail_allocs(count))


def mpzch_launch_count() -> int:
    return int(_lib.mpzch_launch_count())


class MpzchRes:
    """Streaming exporter of fresh rows to a host int8 snapshot (RES)."""

    def __init__(self, table: "MpzchTable", max_rows: int = 0, slots: int = 2,
                 period_ms: int = 15000):
        self.capacity, self.dim = table.capacity, table.dim
        h = C.c_void_p()
        _check("mpzch_res_create", _lib.mpzch_res_create(table.h, max_rows, slots, period_ms,
                                                         C.byref(h)))
        self.h = h

    def stream(self, since_step: int, upto_step: int, stream=None) -> int:
        """Returns MPZCH_OK or MPZCH_EBUSY (every staging slot still in use)."""
        rc = _lib.mpzch_res_stream(self.h, since_step, upto_step, _stream(stream))
        if rc not in (MPZCH_OK, MPZCH_EBUSY):
            raise MpzchError("mpzch_res_stream", rc)
        return rc

    def flush(self, timeout_ms: int = 60000) -> None:
        _check("mpzch_res_flush", _lib.mpzch_res_flush(self.h, timeout_ms))

    def read(self):
        import numpy as np
        keys = np.empty(self.capacity, np.int64)
        q = np.empty((self.capacity, self.dim), np.int8)
        scale = np.empty(self.capacity, np.float32)
        last = np.empty(self.capacity, np.int64)
        ver, upto = C.c_int64(), C.c_int64()
        _check("mpzch_res_read", _lib.mpzch_res_read(
            self.h, keys.ctypes.data_as(C.c_void_p), q.ctypes.data_as(C.c_void_p),
            scale.ctypes.data_as(C.c_void_p), last.ctypes.data_as(C.c_void_p), C.byref(ver),
            C.byref(upto)))
        return keys, q, scale, last, ver.value, upto.value

    def latency(self):
        p50, p99, mx = C.c_double(), C.c_double(), C.c_double()
        n, ovf = C.c_int64(), C.c_int64()
        _check("mpzch_res_latency", _lib.mpzch_res_latency(
            self.h, C.byref(p50), C.byref(p99), C.byref(mx), C.byref(n), C.byref(ovf)))
        return {"p50_ms": p50.value, "p99_ms": p99.value, "max_ms": mx.value,
                "samples": n.value, "overflow_rows": ovf.value}

    def close(self):
        if getattr(self, "h", None):
            _check("mpzch_res_destroy", _lib.mpzch_res_destroy(self.h))
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ handle helper
def _view(addr: int, shape, dtype, device) -> torch.Tensor:
    """A torch tensor over library-owned device memory (no copy, no ownership)."""
    numel = 1
    for s in shape:
        numel *= s
    itemsize = torch.empty((), dtype=dtype).element_size()

    class _Iface:
        __cuda_array_interface__ = {
            "shape": tuple(shape), "typestr": {torch.int64: "<i8", torch.float32: "<f4"}[dtype],
            "data": (addr, False), "version": 3, "strides": None,
        }
    t = torch.as_tensor(_Iface(), device=device)
    assert t.numel() == numel and t.element_size() == itemsize
    return t


def mpzch_owner_partition_workspace(n: int, n_owners: int) -> int:
    b = _lib.mpzch_owner_partition_workspace(n, n_owners)
    if b < 0:
        raise MpzchError("mpzch_owner_partition_workspace", MPZCH_EINVAL)
    return b


def mpzch_owner_partition(ids, n_owners: int, ids_out, pos_out, counts, workspace, src_pos=None,
                          dev_n=None, e=None, e_out=None, stream=None) -> None:
    _need(ids, torch.int64, "ids")
    _need(ids_out, torch.int64, "ids_out")
    _need(pos_out, torch.int32, "pos_out")
    _need(counts, torch.int64, "counts")
    _need(workspace, torch.uint8, "workspace")
    if src_pos is not None:
        _need(src_pos, torch.int32, "src_pos")
    if dev_n is not None:
        _need(dev_n, torch.int64, "dev_n")
    dim = 0
    if e is not None:
        _need(e, torch.float32, "e")
        _need(e_out, torch.float32, "e_out")
        dim = e.shape[1]
        assert e_out.dim() == 2 and e_out.shape[1] == dim
    n = ids.numel()
    assert ids_out.numel() >= n and pos_out.numel() >= n and counts.numel() >= n_owners
    assert e_out is None or e_out.shape[0] >= n
    _check("mpzch_owner_partition", _lib.mpzch_owner_partition(
        _ptr(ids), _ptr(src_pos), n, _ptr(dev_n), n_owners, _ptr(e), dim, _ptr(ids_out),
        _ptr(pos_out), _ptr(e_out), _ptr(counts), _ptr(workspace), workspace.numel(),
        _stream(stream)))


def mpzch_owner_combine(send_ids, pos, n_owners: int, shard_capacity: int, recv_rows, recv_feat,
                        rows, hit, out, ao_table=None, ao_rows=None, status=None, stream=None,
                        n=None) -> None:
    n = send_ids.numel() if n is None else n
    _need(send_ids, torch.int64, "send_ids")
    _need(pos, torch.int32, "pos")
    _need(recv_rows, torch.int32, "recv_rows")
    _need(recv_feat, torch.float32, "recv_feat")
    _need(rows, torch.int32, "rows")
    _need(hit, torch.uint8, "hit")
    _need(out, torch.float32, "out")
    ao_n, ao_dim = 0, 0
    if ao_table is not None:
        _need(ao_table, torch.float32, "ao_table")
        _need(ao_rows, torch.int32, "ao_rows")
        ao_n, ao_dim = ao_table.shape
    if status is not None:
        _need(status, torch.int32, "status")
    assert recv_rows.numel() >= n and recv_feat.dim() == 2 and recv_feat.shape[0] >= n
    _check("mpzch_owner_combine", _lib.mpzch_owner_combine(
        _ptr(send_ids), _ptr(pos), n, n_owners, shard_capacity, _ptr(recv_rows), _ptr(recv_feat),
        recv_feat.shape[1], _ptr(ao_table), ao_n, ao_dim, _ptr(ao_rows), _ptr(rows), _ptr(hit),
        _ptr(out), _ptr(status), _stream(stream)))


class MpzchTable:
    """Owns one table handle; methods forward to the entry points above."""

    def __init__(self, capacity: int, dim: int, probes: int, stream=None, flags: int = 0):
        self.capacity, self.dim, self.probes = capacity, dim, probes
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.h = mpzch_create_ex(capacity, dim, probes, flags, stream)

    def close(self):
        if getattr(self, "h", None):
            mpzch_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def state(self):
        """(keys, last, M) as torch views of the table's own device memory."""
        k, l, m = mpzch_state_views(self.h)
        return (_view(k, (self.capacity,), torch.int64, self.device),
                _view(l, (self.capacity,), torch.int64, self.device),
                _view(m, (self.capacity, self.dim), torch.float32, self.device))

    def lookup(self, ids, rows=None, hit=None, stream=None):
        n = ids.numel()
        rows = torch.empty(n, dtype=torch.int32, device=ids.device) if rows is None else rows
        hit = torch.empty(n, dtype=torch.uint8, device=ids.device) if hit is None else hit
        mpzch_lookup(self.h, ids, rows, hit, stream)
        return rows, hit

    def gather_fused(self, rows, hit, ao_table=None, ao_rows=None, out=None, stream=None):
        n = rows.numel()
        w = self.dim + (0 if ao_table is None else ao_table.shape[1])
        out = torch.empty((n, w), dtype=torch.float32, device=rows.device) if out is None else out
        mpzch_gather_fused(self.h, rows, hit, out, ao_table, ao_rows, stream)
        return out

    def dedup(self, ids, stream=None):
        n = ids.numel()
        uniq = torch.empty(n, dtype=torch.int64, device=ids.device)
        pos = torch.empty(n, dtype=torch.int32, device=ids.device)
        cnt = torch.empty(1, dtype=torch.int64, device=ids.device)
        mpzch_dedup(self.h, ids, uniq, pos, cnt, stream)
        return uniq, pos, cnt

    def writeback(self, ids, e, step, stats=None, stream=None):
        mpzch_writeback(self.h, ids, e, step, stats, stream)

    def train_step(self, ids, n_labeled, e, step, ao_table=None, ao_rows=None, stats=None,
                   inputs_ready=None, stream=None, rows=None, hit=None, out=None):
        dev = ids.device
        w = self.dim + (0 if ao_table is None else ao_table.shape[1])
        rows = torch.empty(n_labeled, dtype=torch.int32, device=dev) if rows is None else rows
        hit = torch.empty(n_labeled, dtype=torch.uint8, device=dev) if hit is None else hit
        out = torch.empty((n_labeled, w), dtype=torch.float32, device=dev) if out is None else out
        mpzch_train_step(self.h, ids, n_labeled, e, step, rows, hit, out, ao_table, ao_rows, stats,
                         inputs_ready, stream)
        return rows, hit, out

    def select_written_since(self, since, stream=None):
        rows = torch.empty(self.capacity, dtype=torch.int32, device=self.device)
        cnt = torch.empty(1, dtype=torch.int64, device=self.device)
        mpzch_select_written_since(self.h, since, rows, cnt, stream)
        return rows, cnt

    def export_int8(self, rows, n=None, dev_n=None, stream=None):
        n = rows.numel() if n is None else n
        q = torch.empty((n, self.dim), dtype=torch.int8, device=self.device)
        scale = torch.empty(n, dtype=torch.float32, device=self.device)
        keys = torch.empty(n, dtype=torch.int64, device=self.device)
        mpzch_export_int8(self.h, rows, q, scale, keys, n=n, dev_n=dev_n, stream=stream)
        return q, scale, keys

    def status(self, stream=None) -> int:
        return mpzch_get_status(self.h, stream)
