"""CPU oracle for the Memory Layer hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg import this package.  The product library never calls it.

This is a thin numpy/ctypes wrapper around ``libmpzch_oracle.so`` (plain
single-threaded C++, see ``mpzch_oracle.cpp`` for the page passages each rule
restates).  Every value this module returns is computed on the host CPU.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import numpy as np

from . import build as _build

ORC_OK = 0
ORC_EINVAL = -1
ORC_ENOMEM = -2
ORC_EBADKEY = -4
ORC_EUNTRACKED = -5

_lib = None


class WbStats(C.Structure):
    _fields_ = [(n, C.c_int64) for n in
                ("n_ids", "n_unique", "n_hit_unique", "n_inserted", "n_evicted", "n_dropped")]

    def as_dict(self):
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


def lib():
    global _lib
    if _lib is None:
        # MPZCH_ORACLE_LIB lets the mutation tests load a deliberately broken
        # copy of the oracle; normally the library is built from this folder.
        path = os.environ.get("MPZCH_ORACLE_LIB") or _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i64, i32 = C.c_int64, C.c_int32
        L.orc_splitmix64.restype = C.c_uint64
        L.orc_splitmix64.argtypes = [C.c_uint64]
        L.orc_home_slot.restype = i64
        L.orc_home_slot.argtypes = [i64, i64]
        L.orc_owner.restype = i32
        L.orc_owner.argtypes = [i64, i32]
        L.orc_owners.argtypes = [p, i64, i32, p]
        L.orc_create.argtypes = [i64, i32, i32, i32, C.POINTER(p)]
        L.orc_destroy.argtypes = [p]
        L.orc_destroy.restype = None
        L.orc_track_rows.argtypes = [p, p, i64]
        L.orc_lookup.argtypes = [p, p, i64, p, p]
        L.orc_gather_fused.argtypes = [p, p, p, i64, p, i64, i32, p, p]
        L.orc_dedup.argtypes = [p, i64, p, p, p]
        L.orc_writeback.argtypes = [p, p, p, i64, i64, p]
        L.orc_set_learning_rate.argtypes = [p, C.c_float]
        L.orc_select_written_since.argtypes = [p, i64, p, p]
        L.orc_quantize_row.argtypes = [p, i32, p, p]
        L.orc_export_int8.argtypes = [p, p, i64, p, p, p]
        L.orc_serve_gather.argtypes = [p, i64, i32, p, p, i32, p, i64, p, p, p]
        L.orc_state.argtypes = [p, p, p, p]
        L.orc_get_row.argtypes = [p, i32, p]
        L.orc_get_rows.argtypes = [p, p, i64, p]
        L.orc_set_row.argtypes = [p, i32, p]
        L.orc_set_state.argtypes = [p, p, p, i64]
        for f in ("orc_create", "orc_track_rows", "orc_lookup", "orc_gather_fused", "orc_dedup",
                  "orc_writeback", "orc_select_written_since", "orc_quantize_row",
                  "orc_export_int8", "orc_serve_gather", "orc_state", "orc_get_row",
                  "orc_set_row", "orc_set_state", "orc_get_rows", "orc_set_learning_rate",
                  "orc_owners"):
            getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def splitmix64(x: int) -> int:
    return int(lib().orc_splitmix64(C.c_uint64(x & ((1 << 64) - 1))))


def home_slot(key: int, capacity: int) -> int:
    return int(lib().orc_home_slot(key, capacity))


def owner(key: int, n_owners: int) -> int:
    return int(lib().orc_owner(key, n_owners))


def owners(ids: np.ndarray, n_owners: int) -> np.ndarray:
    ids = _c(ids, np.int64)
    out = np.empty(ids.size, np.int32)
    rc = lib().orc_owners(_ptr(ids), ids.size, n_owners, _ptr(out))
    assert rc == ORC_OK, rc
    return out


def dedup(ids: np.ndarray):
    ids = _c(ids, np.int64)
    n = ids.size
    uniq = np.empty(n, np.int64)
    pos = np.empty(n, np.int64)
    nu = C.c_int64(0)
    rc = lib().orc_dedup(_ptr(ids), n, _ptr(uniq), _ptr(pos), C.byref(nu))
    assert rc == ORC_OK, rc
    return uniq[:nu.value], pos[:nu.value]


def quantize_row(x: np.ndarray):
    x = _c(x, np.float32)
    q = np.empty(x.size, np.int8)
    s = np.empty(1, np.float32)
    rc = lib().orc_quantize_row(_ptr(x), x.size, _ptr(q), _ptr(s))
    assert rc == ORC_OK, rc
    return q, s[0]


def serve_gather(snap_keys, capacity, probes, snap_q, snap_scale, dim, ids):
    snap_keys = _c(snap_keys, np.int64)
    snap_q = _c(snap_q, np.int8)
    snap_scale = _c(snap_scale, np.float32)
    ids = _c(ids, np.int64)
    n = ids.size
    rows = np.empty(n, np.int32)
    hit = np.empty(n, np.uint8)
    out = np.empty((n, dim), np.float32)
    rc = lib().orc_serve_gather(_ptr(snap_keys), capacity, probes, _ptr(snap_q), _ptr(snap_scale),
                                dim, _ptr(ids), n, _ptr(rows), _ptr(hit), _ptr(out))
    return rc, rows, hit, out


class OracleTable:
    """The oracle's table: identity map + metadata (always full) and value rows
    (all of them, or only a tracked subset for tables too large for host RAM)."""

    def __init__(self, capacity: int, dim: int, probes: int, track_all: bool = True):
        h = C.c_void_p()
        rc = lib().orc_create(capacity, dim, probes, 1 if track_all else 0, C.byref(h))
        if rc != ORC_OK:
            raise ValueError(f"orc_create failed: {rc}")
        self.h = h
        self.capacity, self.dim, self.probes = capacity, dim, probes

    def close(self):
        if self.h:
            lib().orc_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def track_rows(self, rows):
        rows = _c(rows, np.int32)
        rc = lib().orc_track_rows(self.h, _ptr(rows), rows.size)
        assert rc == ORC_OK, rc

    def lookup(self, ids):
        ids = _c(ids, np.int64)
        n = ids.size
        rows = np.empty(n, np.int32)
        hit = np.empty(n, np.uint8)
        rc = lib().orc_lookup(self.h, _ptr(ids), n, _ptr(rows), _ptr(hit))
        return rc, rows, hit

    def gather_fused(self, rows, hit, ao=None, ao_rows=None):
        rows = _c(rows, np.int32)
        hit = _c(hit, np.uint8)
        n = rows.size
        ao_dim = 0 if ao is None else ao.shape[1]
        ao_n = 0 if ao is None else ao.shape[0]
        ao = None if ao is None else _c(ao, np.float32)
        ao_rows = None if ao_rows is None else _c(ao_rows, np.int32)
        out = np.empty((n, self.dim + ao_dim), np.float32)
        rc = lib().orc_gather_fused(self.h, _ptr(rows), _ptr(hit), n, _ptr(ao), ao_n, ao_dim,
                                    _ptr(ao_rows), _ptr(out))
        assert rc == ORC_OK, rc
        return out

    def writeback(self, ids, e, step):
        ids = _c(ids, np.int64)
        e = _c(e, np.float32)
        assert e.shape == (ids.size, self.dim), (e.shape, ids.size, self.dim)
        st = WbStats()
        rc = lib().orc_writeback(self.h, _ptr(ids), _ptr(e), ids.size, step, C.byref(st))
        return rc, st.as_dict()

    def set_learning_rate(self, eta):
        rc = lib().orc_set_learning_rate(self.h, float(eta))
        assert rc == ORC_OK, rc

    def select_written_since(self, since):
        out = np.empty(self.capacity, np.int32)
        cnt = C.c_int64(0)
        rc = lib().orc_select_written_since(self.h, since, _ptr(out), C.byref(cnt))
        assert rc == ORC_OK, rc
        return out[:cnt.value].copy()

    def export_int8(self, rows):
        rows = _c(rows, np.int32)
        n = rows.size
        q = np.empty((n, self.dim), np.int8)
        s = np.empty(n, np.float32)
        k = np.empty(n, np.int64)
        rc = lib().orc_export_int8(self.h, _ptr(rows), n, _ptr(q), _ptr(s), _ptr(k))
        assert rc == ORC_OK, rc
        return q, s, k

    def state(self):
        """(keys, last) as numpy copies, and the last step."""
        kp = C.POINTER(C.c_int64)()
        lp = C.POINTER(C.c_int64)()
        ls = C.c_int64(0)
        rc = lib().orc_state(self.h, C.byref(kp), C.byref(lp), C.byref(ls))
        assert rc == ORC_OK, rc
        keys = np.ctypeslib.as_array(kp, shape=(self.capacity,)).copy()
        last = np.ctypeslib.as_array(lp, shape=(self.capacity,)).copy()
        return keys, last, ls.value

    def row(self, r):
        out = np.empty(self.dim, np.float32)
        rc = lib().orc_get_row(self.h, int(r), _ptr(out))
        assert rc == ORC_OK, rc
        return out

    def rows(self, rs):
        rs = _c(rs, np.int32)
        out = np.empty((rs.size, self.dim), np.float32)
        rc = lib().orc_get_rows(self.h, _ptr(rs), rs.size, _ptr(out))
        assert rc == ORC_OK, rc
        return out

    def set_row(self, r, x):
        x = _c(x, np.float32)
        rc = lib().orc_set_row(self.h, int(r), _ptr(x))
        assert rc == ORC_OK, rc

    def set_state(self, keys, last, last_step):
        keys = _c(keys, np.int64)
        last = _c(last, np.int64)
        rc = lib().orc_set_state(self.h, _ptr(keys), _ptr(last), last_step)
        assert rc == ORC_OK, rc

    def values(self):
        """Dense copy of every value row (track_all tables only)."""
        return self.rows(np.arange(self.capacity, dtype=np.int32))


def oracle_lib_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmpzch_oracle.so")


class ShardedOracle:
    """Hash-owner sharding of the table over G shards, one per rank.

    Memory Layer section 2 shards the table across devices and keeps the
    distributed lookup's all-to-all exchange; MTGR section 3.3 exchanges ids
    all-to-all and dedups twice, before and after the exchange.  Key k lives
    in shard owner(k) = (splitmix64(k) >> 32) mod G, an ordinary oracle table
    of `shard_capacity` rows.  Global row of shard s, local row r: s*C_s + r.

    One step, for the batches of ranks 0..G-1:
      1. each rank's labeled ids are looked up (and gathered, with the
         rank's always-on rows) at their owners, on the tables as they were
         before the step;
      2. each rank dedups its whole batch (first occurrence keeps its e row),
         sends each distinct id with its e row to its owner; an owner receives
         the ids of ranks 0..G-1 in rank order, each rank's in batch order, and
         runs the Writeback on that batch, which dedups again.
    """

    def __init__(self, n_shards: int, shard_capacity: int, dim: int, probes: int):
        self.G, self.Cs, self.dim, self.probes = n_shards, shard_capacity, dim, probes
        self.shards = [OracleTable(shard_capacity, dim, probes) for _ in range(n_shards)]

    def close(self):
        for t in self.shards:
            t.close()

    def lookup_gather(self, ids, ao=None, ao_rows=None):
        """Rows (global), hit and gathered features of one rank's labeled ids."""
        ids = _c(ids, np.int64)
        n = ids.size
        own = owners(ids, self.G)
        rows = np.full(n, -1, np.int32)
        hit = np.zeros(n, np.uint8)
        width = self.dim + (0 if ao is None else ao.shape[1])
        out = np.zeros((n, width), np.float32)
        rc_all = ORC_OK
        for s in range(self.G):
            at = np.nonzero(own == s)[0]
            if at.size == 0:
                continue
            rc, r, h = self.shards[s].lookup(ids[at])
            rc_all = rc_all or rc
            out[at] = self.shards[s].gather_fused(r, h, ao, None if ao_rows is None else ao_rows[at])
            rows[at] = np.where(h != 0, r + s * self.Cs, -1)
            hit[at] = h
        return rc_all, rows, hit, out

    def routed_batches(self, rank_ids, rank_e):
        """What each owner receives: (ids, e) per shard after the first dedup."""
        recv_ids = [[] for _ in range(self.G)]
        recv_e = [[] for _ in range(self.G)]
        for ids, e in zip(rank_ids, rank_e):  # ranks in order
            uniq, pos = dedup(ids)
            own = owners(uniq, self.G)
            for s in range(self.G):
                sel = own == s
                recv_ids[s].append(uniq[sel])
                recv_e[s].append(_c(e, np.float32)[pos[sel]])
        return ([np.concatenate(x) for x in recv_ids],
                [np.concatenate(x).reshape(-1, self.dim) for x in recv_e])

    def writeback(self, rank_ids, rank_e, step):
        """Per-shard (rc, stats) of the step's Writeback."""
        recv_ids, recv_e = self.routed_batches(rank_ids, rank_e)
        return [self.shards[s].writeback(recv_ids[s], recv_e[s], step) for s in range(self.G)]

    def state(self, s):
        return self.shards[s].state()

    def values(self, s):
        return self.shards[s].values()

