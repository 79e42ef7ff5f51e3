"""The C ABI without a GPU: the library builds for sm_100a, loads, exports every
entry point the header declares, and rejects bad arguments on the host before
any CUDA call is made (including a simulated allocation failure)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mpzch.h")


@pytest.fixture(scope="module")
def lib():
    from hashed_sparse_table_b200 import build
    path = build.build()
    return C.CDLL(path)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MPZCH_API\s+\w+\s+(mpzch_\w+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    syms = declared_symbols()
    for name in ("mpzch_create", "mpzch_destroy", "mpzch_lookup", "mpzch_gather_fused",
                 "mpzch_writeback", "mpzch_export_int8", "mpzch_select_written_since",
                 "mpzch_serve_gather", "mpzch_dedup", "mpzch_get_status", "mpzch_state_views"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    path = lib._name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (mpzch_\w+)", out))
    assert set(declared_symbols()) <= exported
    # nothing but the declared API is exported under the library's prefix
    assert exported <= set(declared_symbols())


def _setup(lib):
    p, i64, i32 = C.c_void_p, C.c_int64, C.c_int32
    lib.mpzch_create.argtypes = [i64, i32, i32, p, C.POINTER(p)]
    lib.mpzch_debug_fail_allocs.argtypes = [i32]
    lib.mpzch_lookup.argtypes = [p, p, i64, p, p, p]
    lib.mpzch_writeback.argtypes = [p, p, p, i64, i64, p, p]
    lib.mpzch_serve_gather.argtypes = [p, i64, i32, p, p, i32, p, i64, p, p, p, p, p]
    lib.mpzch_set_option.argtypes = [p, i32, i64]
    lib.mpzch_gather_fused.argtypes = [p, p, p, i64, p, i64, i32, p, p, p]
    lib.mpzch_export_int8.argtypes = [p, p, i64, p, p, p, p, p]
    lib.mpzch_dedup.argtypes = [p, p, i64, p, p, p, p]
    return p


@pytest.mark.parametrize("cap,dim,probes", [
    (0, 64, 4), (-5, 64, 4), (1 << 31, 64, 4), (4096, 0, 4), (4096, 6, 4), (4096, 64, 0),
    (4096, 64, 4097), (16, 8, 17),
])
def test_create_rejects_bad_sizes_without_touching_the_gpu(lib, cap, dim, probes):
    p = _setup(lib)
    h = p()
    assert lib.mpzch_create(cap, dim, probes, None, C.byref(h)) == -1
    assert not h.value


def test_create_null_out(lib):
    _setup(lib)
    assert lib.mpzch_create(16, 4, 2, None, None) == -1


def test_create_reports_enomem_from_allocation_hook(lib):
    p = _setup(lib)
    h = p()
    assert lib.mpzch_debug_fail_allocs(1) == 0
    assert lib.mpzch_create(1 << 20, 512, 8, None, C.byref(h)) == -2
    assert not h.value
    assert lib.mpzch_debug_fail_allocs(-1) == -1


def test_calls_on_null_table_are_einval(lib):
    _setup(lib)
    assert lib.mpzch_lookup(None, None, 0, None, None, None) == -1
    assert lib.mpzch_writeback(None, None, None, 0, 0, None, None) == -1
    assert lib.mpzch_set_option(None, 1, 3) == -1
    assert lib.mpzch_gather_fused(None, None, None, 0, None, 0, 0, None, None, None) == -1
    assert lib.mpzch_export_int8(None, None, 0, None, None, None, None, None) == -1
    assert lib.mpzch_dedup(None, None, 0, None, None, None, None) == -1
    assert lib.mpzch_destroy(None) == 0


@pytest.mark.parametrize("cap,probes,dim,n", [
    (0, 1, 4, 1), (8, 9, 4, 1), (8, 0, 4, 1), (8, 2, 6, 1), (8, 2, 0, 1), (8, 2, 4, -1),
])
def test_serve_gather_rejects_bad_sizes(lib, cap, probes, dim, n):
    _setup(lib)
    assert lib.mpzch_serve_gather(None, cap, probes, None, None, dim, None, n, None, None, None,
                                  None, None) == -1


def test_serve_gather_rejects_null_buffers_and_accepts_empty(lib):
    _setup(lib)
    assert lib.mpzch_serve_gather(None, 8, 2, None, None, 4, None, 3, None, None, None, None,
                                  None) == -1
    assert lib.mpzch_serve_gather(None, 8, 2, None, None, 4, None, 0, None, None, None, None,
                                  None) == 0


def test_res_create_rejects_bad_arguments(lib):
    p = _setup(lib)
    lib.mpzch_res_create.argtypes = [p, C.c_int64, C.c_int32, C.c_int32, C.POINTER(p)]
    h = p()
    assert lib.mpzch_res_create(None, 0, 2, 100, C.byref(h)) == -1
    assert lib.mpzch_res_create(None, 0, 2, 100, None) == -1
    lib.mpzch_res_stream.argtypes = [p, C.c_int64, C.c_int64, p]
    assert lib.mpzch_res_stream(None, 0, 0, None) == -1
    lib.mpzch_res_flush.argtypes = [p, C.c_int32]
    assert lib.mpzch_res_flush(None, 10) == -1
    lib.mpzch_res_destroy.argtypes = [p]
    assert lib.mpzch_res_destroy(None) == 0


def test_python_binding_loads(lib):
    from hashed_sparse_table_b200 import binding
    assert binding.mpzch_launch_count() >= 0
    with pytest.raises(binding.MpzchError):
        binding.mpzch_debug_fail_allocs(-3)


def test_owner_partition_and_combine_reject_bad_arguments_without_the_gpu(lib):
    p, i64, i32 = C.c_void_p, C.c_int64, C.c_int32
    lib.mpzch_owner_partition_workspace.argtypes = [i64, i32]
    lib.mpzch_owner_partition_workspace.restype = i64
    assert lib.mpzch_owner_partition_workspace(0, 1) == 0
    assert lib.mpzch_owner_partition_workspace(1, 1) == 256
    assert lib.mpzch_owner_partition_workspace(163840, 8) == 160 * 8 * 4  # 1024-id tiles
    for n, g in ((-1, 4), (10, 0), (10, 257), (1 << 31, 4)):
        assert lib.mpzch_owner_partition_workspace(n, g) == -1
    lib.mpzch_owner_partition.argtypes = [p, p, i64, p, i32, p, i32, p, p, p, p, p, i64, p]
    fake = C.c_void_p(0x1000)
    # bad owner counts, missing counts, missing buffers, short workspace, odd dim
    assert lib.mpzch_owner_partition(fake, None, 10, None, 0, None, 0, fake, fake, None, fake,
                                     fake, 4096, None) == -1
    assert lib.mpzch_owner_partition(fake, None, 10, None, 4, None, 0, fake, fake, None, None,
                                     fake, 4096, None) == -1
    assert lib.mpzch_owner_partition(fake, None, 10, None, 4, None, 0, None, fake, None, fake,
                                     fake, 4096, None) == -1
    assert lib.mpzch_owner_partition(fake, None, 10, None, 4, None, 0, fake, fake, None, fake,
                                     fake, 16, None) == -1
    assert lib.mpzch_owner_partition(fake, None, 10, None, 4, fake, 6, fake, fake, fake, fake,
                                     fake, 4096, None) == -1
    lib.mpzch_owner_combine.argtypes = [p, p, i64, i32, i64, p, p, i32, p, i64, i32, p, p, p, p,
                                        p, p]
    def comb(n=10, G=4, cs=1000, dim=16, ao=None, ao_n=0, ao_dim=0, aor=None, out=fake):
        return lib.mpzch_owner_combine(fake, fake, n, G, cs, fake, fake, dim, ao, ao_n, ao_dim,
                                       aor, fake, fake, out, None, None)
    assert comb(G=0) == -1 and comb(G=257) == -1
    assert comb(cs=1 << 30, G=4) == -1      # global rows would pass 2^31
    assert comb(dim=6) == -1
    assert comb(ao=fake, ao_n=5, ao_dim=8, aor=None) == -1
    assert comb(ao=None, ao_dim=8) == -1
    assert comb(out=None) == -1
    assert comb(n=0) == 0                   # nothing to do, nothing launched
