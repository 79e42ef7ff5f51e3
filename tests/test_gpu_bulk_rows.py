"""Bulk-copy row kernels (MPZCH_OPT_ROW_KERNEL = 1) vs the CPU oracle, bit for bit.

The fused gather and the Writeback row update move rows through shared memory
with 1-D bulk copies completed on mbarriers instead of through registers.
Their results must be exactly those of the register kernels, i.e. of the
oracle: gathered features (cached row or +0, always-on concat), and the table
values after every step.  Cases: the scaled workloads with separate calls,
the fused step and pipelined steps; every launch shape (warps per block,
blocks per SM) and L2 hint; rows too large for one warp's stages (the
register kernel runs); tiny rows; out-of-range rows in the gather.
"""
import numpy as np
import pytest
import torch

from hashed_sparse_table_b200 import inputs
from gpu_harness import run_pair, run_pipelined
from test_gpu_parity import CLUSTERED, SCALED

pytestmark = pytest.mark.gpu


def _opts(**kw):
    from hashed_sparse_table_b200 import binding
    o = {binding.MPZCH_OPT_ROW_KERNEL: 1}
    names = {"warps": binding.MPZCH_OPT_BULK_WARPS, "blocks": binding.MPZCH_OPT_BULK_BLOCKS,
             "hint": binding.MPZCH_OPT_L2_HINT_ROWS}
    for k, v in kw.items():
        o[names[k]] = v
    return o


def test_bulk_tiny_workload_bit_exact():
    run_pair(inputs.CFG1_TINY, options=_opts())


@pytest.mark.parametrize("name", ["c2_small", "c3_small", "c4_stress", "nonpow2", "p_eq_c",
                                  "tiny_table"])
@pytest.mark.parametrize("fused", [False, True])
def test_bulk_scaled_workloads_bit_exact(name, fused):
    run_pair(SCALED[name], fused_step=fused, options=_opts())


@pytest.mark.parametrize("name", ["c3_small", "c4_stress"])
def test_bulk_pipelined_steps_bit_exact(name):
    run_pipelined(SCALED[name], options=_opts())


def test_bulk_pipelined_cluster_placement_bit_exact():
    run_pipelined(CLUSTERED["clus_p8"], options=_opts())


@pytest.mark.parametrize("warps,blocks,hint", [(1, 1, 0), (2, 3, 1), (4, 2, 2), (16, 1, 0),
                                               (8, 8, 1)])
def test_bulk_launch_shapes_and_hints_bit_exact(warps, blocks, hint):
    run_pair(SCALED["c3_small"].scaled(steps=6), fused_step=True,
             options=_opts(warps=warps, blocks=blocks, hint=hint))


@pytest.mark.parametrize("dim", [4, 2048, 8192])
def test_bulk_row_sizes_bit_exact(dim):
    """dim 4: 16-byte rows; 2048: fewer warps per block so the stages fit;
    8192: too large for one warp's stages, the register kernel runs."""
    w = inputs.Workload(f"bulk_d{dim}", 21, capacity=512, dim=dim, probes=4, steps=5,
                        labeled=300, pool=100, zipf_alpha=1.05, zipf_keys=3_000, ao_rows=64,
                        ao_dim=8, ao_kind="mod")
    run_pair(w, fused_step=True, options=_opts())


def test_bulk_learning_rate_bit_exact():
    run_pair(SCALED["c3_small"].scaled(steps=6), eta=0.5, options=_opts())


def test_bulk_gather_bad_rows_set_status_and_give_zeros():
    from hashed_sparse_table_b200 import binding
    tbl = binding.MpzchTable(128, 8, 4)
    binding.mpzch_set_option(tbl.h, binding.MPZCH_OPT_ROW_KERNEL, 1)
    dev = tbl.device
    rows = torch.tensor([0, 500, -3, 7], dtype=torch.int32, device=dev)
    hit = torch.tensor([1, 1, 1, 0], dtype=torch.uint8, device=dev)
    ao = torch.arange(16 * 4, dtype=torch.float32, device=dev).view(16, 4)
    aor = torch.tensor([1, 2, 99, 3], dtype=torch.int32, device=dev)
    out = tbl.gather_fused(rows, hit, ao, aor)
    st = tbl.status()
    assert st & binding.MPZCH_STATUS_BADROW and st & binding.MPZCH_STATUS_BADAO
    assert not st & binding.MPZCH_STATUS_TIMEOUT
    o = out.cpu().numpy()
    assert (o[1:3, :8] == 0).all() and (o[2, 8:] == 0).all()
    assert (o[0, 8:] == np.arange(4, 8)).all() and (o[3, 8:] == np.arange(12, 16)).all()
    assert (o[0, :8] == 0).all()  # the empty table's row 0 holds zeros
