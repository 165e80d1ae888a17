"""The allocation-free mask entry point gives the same routing as the
workspace one.

sba_build_mask_noalloc exists for callers that cannot allocate device memory
or hand the library a workspace (plugin interfaces that pass only inputs and
outputs; services that reserve all device memory at start-up and forbid later
cudaMalloc). It keeps its scratch in the library's static device array, so
this test runs two different layers through it back to back: the second call
must not see anything the first one left behind. The mask is integer data, so
the comparison is bit-exact. This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import datagen

pytestmark = pytest.mark.gpu


def _routing(sba, wl, use_noalloc):
    dev = torch.device("cuda:0")
    q, k, v = datagen.generate(wl, seed=3, device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube)
    sa = sba.SparseAttention(plan, device=dev)
    sba.sba_reorder(plan.handle, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace)
    args = (plan.handle, sa.qt, sa.kt, wl.top_p_per_head(), wl.top_k, sa.bitmask, sa.row_cnt,
            sa.row_ptr, sa.col_idx)
    if use_noalloc:
        sba.sba_build_mask_noalloc(*args, sa.work_order)
    else:
        sba.sba_build_mask(*args, sa.work_order, sa.workspace)
    torch.cuda.synchronize()
    nnz = int(sa.row_ptr[-1].item())
    return {"bitmask": sa.bitmask.cpu().numpy(), "row_cnt": sa.row_cnt.cpu().numpy(),
            "row_ptr": sa.row_ptr.cpu().numpy(), "col_idx": sa.col_idx[:nnz].cpu().numpy(),
            "work_order": sa.work_order.cpu().numpy()}


def test_noalloc_mask_equals_workspace_mask_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_sba_b200 as sba
    layers = [
        datagen.custom("noalloc_a", 1, 3, 5, 20, 19, 128, (2, 8, 8), top_p=(0.8, 0.9, 0.95),
                       top_k=3, rope_split=(44, 42, 42)),
        datagen.custom("noalloc_b", 2, 2, 8, 16, 16, 64, (4, 4, 4), top_p=(0.6, 0.9), top_k=2,
                       rope_split=(16, 24, 24)),
    ]
    ref = [_routing(sba, wl, use_noalloc=False) for wl in layers]
    got = [_routing(sba, wl, use_noalloc=True) for wl in layers]  # two calls in a row
    for r, g in zip(ref, got):
        for key in r:
            assert np.array_equal(r[key], g[key]), key
    # the device-side checks of those calls found nothing, and reading the
    # status clears it
    assert sba.sba_noalloc_status() == sba.SBA_OK
    assert sba.sba_noalloc_status() == sba.SBA_OK


def test_noalloc_rejects_a_plan_larger_than_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_sba_b200 as sba
    plan = sba.Plan(1, 64, 33, 45, 80, 128, (2, 8, 8), "bf16")  # 64 heads x 1020 blocks x 128
    fake = 1 << 20  # rejected before any device access
    with pytest.raises(sba.SbaError) as e:
        sba.sba_build_mask_noalloc(plan.handle, fake, fake, [0.9] * 64, 8, fake, fake, fake, fake,
                                   fake)
    assert e.value.status == sba.SBA_ERR_CAPACITY
    assert "scratch" in sba.sba_last_error()


def test_a_failed_call_is_not_remembered():
    """A call that fails (here an unaligned input, rejected before any device
    access) leaves nothing behind: the next good call succeeds, its error
    text is empty and its routing equals the workspace path's."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_sba_b200 as sba
    wl = datagen.custom("noalloc_c", 1, 2, 5, 20, 19, 128, (2, 8, 8), top_p=(0.85, 0.9), top_k=2,
                        rope_split=(44, 42, 42))
    dev = torch.device("cuda:0")
    q, k, v = datagen.generate(wl, seed=4, device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube)
    sa = sba.SparseAttention(plan, device=dev)
    with pytest.raises(sba.SbaError) as e:
        sba.sba_build_mask_noalloc(plan.handle, sa.qt.data_ptr() + 2, sa.kt, wl.top_p_per_head(),
                                   wl.top_k, sa.bitmask, sa.row_cnt, sa.row_ptr, sa.col_idx,
                                   sa.work_order)
    assert e.value.status == sba.SBA_ERR_INVALID_ARG
    ref = _routing(sba, wl, use_noalloc=False)
    got = _routing(sba, wl, use_noalloc=True)
    assert sba.sba_last_error() == ""
    for key in ref:
        assert np.array_equal(ref[key], got[key]), key
    assert sba.sba_noalloc_status() == sba.SBA_OK
