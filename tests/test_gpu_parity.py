"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the same
seeded inputs: small workloads element by element, full-size workloads on
sampled query blocks plus exact bookkeeping, and the edge cases."""
import math

import numpy as np
import pytest
import torch

import datagen
import oracle
from parity_utils import (ATOL, REL_L2, attention_errors, compare_mask, geom_of,
                          oracle_attention_blocks, oracle_mask_per_head, run_gpu, sample_blocks, to64)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": datagen.WORKLOADS["tiny"],
    "small": datagen.WORKLOADS["small"],
    # ragged grids in every axis, several tiles and a ragged tail
    "ragged_d128_bs128": datagen.custom("ragged_d128_bs128", 1, 3, 5, 20, 19, 128, (2, 8, 8),
                                        top_p=(0.8, 0.9, 0.95), top_k=3, rope_split=(44, 42, 42)),
    "ragged_d64_bs128": datagen.custom("ragged_d64_bs128", 2, 2, 3, 9, 17, 64, (2, 8, 8),
                                       top_p=(0.7, 0.9), top_k=2, rope_split=(16, 24, 24)),
    "ragged_d128_bs64": datagen.custom("ragged_d128_bs64", 1, 2, 6, 10, 10, 128, (1, 8, 8),
                                       top_p=(0.85,), top_k=2, rope_split=(44, 42, 42)),
    "ragged_f32": datagen.custom("ragged_f32", 1, 2, 5, 6, 7, 64, (4, 4, 4), dtype="f32",
                                 top_p=(0.9,), top_k=1),
    # Hilbert-curve block organisation (ragged tail block, both tile shapes)
    "hilbert_d128_bs128": datagen.custom("hilbert_d128_bs128", 1, 3, 5, 20, 19, 128, (2, 8, 8),
                                         top_p=(0.8, 0.9, 0.95), top_k=3, rope_split=(44, 42, 42),
                                         order="hilbert"),
    "hilbert_small": datagen.with_order(datagen.WORKLOADS["small"], "hilbert"),
    "hilbert_f32": datagen.custom("hilbert_f32", 1, 2, 5, 6, 7, 64, (4, 4, 4), dtype="f32",
                                  top_p=(0.9,), top_k=1, order="hilbert"),
    # 1080 rows (40 heads x 27 blocks, ragged in h and w): several rows per
    # persistent CTA, so a CTA goes through many row changes
    "many_rows_d128": datagen.custom("many_rows_d128", 1, 40, 6, 22, 21, 128, (2, 8, 8),
                                     top_p=(0.5, 0.9, 0.97), top_k=2, rope_split=(44, 42, 42)),
    # block size 64 with an odd number of blocks per head (27): the last pair
    # of query blocks has no second block; corner cubes hold a single token
    "pairs_odd_bs64": datagen.custom("pairs_odd_bs64", 1, 2, 3, 17, 17, 128, (1, 8, 8),
                                     top_p=(0.7, 0.9), top_k=2, rope_split=(44, 42, 42)),
    "pairs_odd_d64": datagen.custom("pairs_odd_d64", 2, 2, 9, 12, 12, 64, (4, 4, 4),
                                    top_p=(0.6, 0.95), top_k=1, rope_split=(16, 24, 24)),
}


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


_cache = {}


def _inputs(name, wl):
    if name not in _cache:
        dev = _cuda()
        _cache[name] = datagen.generate(wl, seed=0, device=dev)
    return _cache[name]


@pytest.fixture(scope="module", params=list(SMALL))
def small_case(request):
    name = request.param
    wl = SMALL[name]
    q, k, v = _inputs(name, wl)
    gpu = run_gpu(wl, q, k, v)
    return name, wl, (q, k, v), gpu


def test_reorder_and_unreorder_bit_exact(small_case):
    name, wl, (q, k, v), gpu = small_case
    g = geom_of(wl)
    for x, xt in ((q, gpu["qt"]), (k, gpu["kt"]), (v, gpu["vt"])):
        assert np.array_equal(to64(xt), oracle.reorder(to64(x.cpu()), g))
    assert np.array_equal(to64(gpu["o"]), oracle.unreorder(to64(gpu["ot"]), g))
    assert gpu["status"] == 0


def test_mask_matches_oracle(small_case):
    name, wl, _, gpu = small_case
    g = geom_of(wl)
    orc = oracle_mask_per_head(wl, to64(gpu["qt"]), to64(gpu["kt"]), wl.top_p_per_head(), wl.top_k)
    stats = compare_mask(gpu, orc, wl.top_p_per_head(), wl.top_k, g.nb, wl.H)
    print(name, stats)


def test_attention_matches_oracle(small_case):
    name, wl, _, gpu = small_case
    g = geom_of(wl)
    Ot, lse = oracle.attention(to64(gpu["qt"]), to64(gpu["kt"]), to64(gpu["vt"]), g,
                               gpu["row_ptr"], gpu["col_idx"])
    valid = oracle.slot_valid(g)
    got = to64(gpu["ot"])
    assert np.all(got[:, :, ~valid] == 0)
    mx, rel = attention_errors(got[:, :, valid], Ot[:, :, valid])
    print(name, "max-abs", mx, "rel-L2", rel)
    assert mx <= ATOL and rel <= REL_L2
    lerr = np.abs(gpu["lse"].double().numpy()[:, :, valid] - lse[:, :, valid]).max()
    assert lerr <= 1e-2, lerr


def test_end_to_end_against_oracle_forward(small_case):
    """Raster output vs the oracle's own forward pass on the query blocks
    whose routing agrees (all of them, unless a boundary row differs)."""
    name, wl, (q, k, v), gpu = small_case
    g = geom_of(wl)
    o_ref, m, _ = oracle.forward(to64(q.cpu()), to64(k.cpu()), to64(v.cpu()), g,
                                 wl.top_p_per_head(), wl.top_k)
    same = np.array([np.array_equal(gpu["col_idx"][gpu["row_ptr"][r]:gpu["row_ptr"][r + 1]],
                                    m["col_idx"][m["row_ptr"][r]:m["row_ptr"][r + 1]])
                     for r in range(gpu["row_cnt"].size)]).reshape(wl.B, wl.H, g.nb)
    blk = oracle.slot_of_token(g) // g.bs
    keep = same[:, :, blk]  # [B,H,N]
    mx, rel = attention_errors(to64(gpu["o"])[keep], o_ref[keep])
    assert keep.mean() > 0.9 and mx <= ATOL and rel <= REL_L2


def test_lpt_and_head_major_schedules_agree_bitwise(small_case):
    name, wl, (q, k, v), gpu = small_case
    hm = run_gpu(wl, q, k, v, sched=1)
    assert torch.equal(hm["ot"], gpu["ot"]) and torch.equal(hm["lse"], gpu["lse"])


def test_strided_raster_layout():
    """q/k/v/o stored as [B, N, H, d] (heads interleaved) give the same result."""
    wl = SMALL["ragged_d64_bs128"]
    q, k, v = _inputs("ragged_d64_bs128", wl)
    base = run_gpu(wl, q, k, v)
    qs, ks, vs = (x.transpose(1, 2).contiguous().transpose(1, 2) for x in (q, k, v))
    assert qs.stride(2) == wl.H * wl.d
    alt = run_gpu(wl, qs, ks, vs)
    assert torch.equal(alt["qt"], base["qt"]) and torch.equal(alt["ot"], base["ot"])
    assert torch.equal(alt["o"], base["o"])


def test_p1_is_dense_attention():
    wl = SMALL["ragged_d128_bs128"]
    q, k, v = _inputs("ragged_d128_bs128", wl)
    g = geom_of(wl)
    gpu = run_gpu(wl, q, k, v, top_p=[1.0] * wl.H, top_k=1)
    assert np.all(gpu["row_cnt"] == g.nb)
    qt, kt, vt = (to64(gpu[x]) for x in ("qt", "kt", "vt"))
    valid = torch.from_numpy(oracle.slot_valid(g))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qt), torch.from_numpy(kt), torch.from_numpy(vt),
        attn_mask=valid[None, None, None, :]).numpy()
    mx, rel = attention_errors(to64(gpu["ot"])[:, :, valid.numpy()], ref[:, :, valid.numpy()])
    assert mx <= ATOL and rel <= REL_L2


def test_topk_floor_and_cap():
    wl = SMALL["small"]
    q, k, v = _inputs("small", wl)
    g = geom_of(wl)
    gpu = run_gpu(wl, q, k, v, top_p=[1e-6] * wl.H, top_k=3)
    assert np.all(gpu["row_cnt"] == 3)
    orc = oracle_mask_per_head(wl, to64(gpu["qt"]), to64(gpu["kt"]), [1e-6] * wl.H, 3)
    compare_mask(gpu, orc, [1e-6] * wl.H, 3, g.nb, wl.H)
    gpu2 = run_gpu(wl, q, k, v, top_p=[0.5] * wl.H, top_k=g.nb + 7)
    assert np.all(gpu2["row_cnt"] == g.nb)


def _attn_with_csr(wl, q, k, v, row_ptr, col_idx, sched=1, work_counts=None):
    """sba_attention on a hand-made CSR; col_idx is held in a buffer of the
    plan's max_nnz capacity (zero beyond the given entries)."""
    import block_sparse_attention_sba_b200 as sba
    g = geom_of(wl)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube, order=wl.order)
    sa = sba.SparseAttention(plan, device=q.device)
    sba.sba_reorder(plan.handle, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace)
    rp = torch.tensor(row_ptr, dtype=torch.int32, device=q.device)
    ci = torch.zeros(plan.info.max_nnz, dtype=torch.int32, device=q.device)
    if len(col_idx):
        ci[:len(col_idx)] = torch.tensor(col_idx, dtype=torch.int32, device=q.device)
    counts = np.diff(row_ptr) if work_counts is None else work_counts
    wo = torch.tensor(oracle.lpt_order(counts, g.nb), dtype=torch.int32, device=q.device)
    sba.sba_attention(plan.handle, sa.qt, sa.kt, sa.vt, rp, ci, wo, sa.ot, sa.lse, sched, None,
                      sa.workspace)
    torch.cuda.synchronize()
    return sa, sa.check()


@pytest.mark.parametrize("name", ["ragged_d128_bs64", "pairs_odd_bs64", "ragged_d128_bs128",
                                  "ragged_d64_bs128"])
@pytest.mark.parametrize("sched", [0, 1])
def test_handmade_csr_with_empty_and_single_block_rows(sched, name):
    wl = SMALL[name]
    q, k, v = _inputs(name, wl)
    g = geom_of(wl)
    R = wl.B * wl.H * g.nb
    rng = np.random.default_rng(5)
    cols, cnt = [], []
    for r in range(R):
        n = [0, 1, g.nb, int(rng.integers(1, g.nb))][r % 4]
        sel = np.sort(rng.choice(g.nb, size=n, replace=False))
        cols.append(sel)
        cnt.append(n)
    row_ptr = np.concatenate([[0], np.cumsum(cnt)])
    col_idx = np.concatenate(cols)
    sa, status = _attn_with_csr(wl, q, k, v, row_ptr, col_idx, sched)
    assert status == 0
    qt, kt, vt = (to64(x.cpu()) for x in (sa.qt, sa.kt, sa.vt))
    valid = oracle.slot_valid(g)
    got = to64(sa.ot.cpu())
    lse = sa.lse.cpu().double().numpy()
    nonempty = [(b, h, i) for b in range(wl.B) for h in range(wl.H) for i in range(g.nb)
                if cnt[(b * wl.H + h) * g.nb + i] > 0]
    Ot, lref = oracle.attention(qt, kt, vt, g, row_ptr, col_idx, blocks=nonempty)
    for (b, h, i) in nonempty:
        sl = slice(i * g.bs, (i + 1) * g.bs)
        m = valid[sl]
        mx, rel = attention_errors(got[b, h, sl][m], Ot[b, h, sl][m])
        assert mx <= ATOL and rel <= REL_L2
        assert np.abs(lse[b, h, sl][m] - lref[b, h, sl][m]).max() <= 1e-2
    for r in range(R):
        if cnt[r] == 0:
            b, h, i = r // (wl.H * g.nb), (r // g.nb) % wl.H, r % g.nb
            sl = slice(i * g.bs, (i + 1) * g.bs)
            assert np.all(got[b, h, sl] == 0)
            assert np.all(np.isneginf(lse[b, h, sl][valid[sl]]))


@pytest.mark.parametrize("name", ["small", "ragged_d128_bs128"])
def test_out_of_range_column_sets_device_check_and_context_survives(name):
    wl = SMALL[name]
    q, k, v = _inputs(name, wl)
    g = geom_of(wl)
    R = wl.B * wl.H * g.nb
    row_ptr = np.arange(R + 1)
    col_idx = np.zeros(R, dtype=np.int64)
    col_idx[7] = g.nb + 100
    col_idx[9] = -3
    import block_sparse_attention_sba_b200 as sba
    sa, status = _attn_with_csr(wl, q, k, v, row_ptr, col_idx, sched=0)
    assert status == sba.SBA_ERR_DEVICE_CHECK
    sa2, status2 = _attn_with_csr(wl, q, k, v, row_ptr, np.zeros(R, dtype=np.int64), sched=0)
    assert status2 == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["small", "ragged_d128_bs128"])
@pytest.mark.parametrize("sched", [0, 1])
def test_corrupt_row_pointers_are_skipped_and_flagged(name, sched):
    """Row pointers that give a negative length, more than nb columns or a
    start past the plan's col_idx capacity make their rows empty and set
    SBA_ERR_DEVICE_CHECK; every other row is still computed, and nothing is
    read outside the col_idx buffer (it holds max_nnz entries)."""
    wl = SMALL[name]
    q, k, v = _inputs(name, wl)
    g = geom_of(wl)
    R = wl.B * wl.H * g.nb
    row_ptr = np.arange(R + 1, dtype=np.int64)
    col_idx = np.arange(R, dtype=np.int64) % g.nb
    good_counts = np.ones(R, dtype=np.int64)
    row_ptr[5] = row_ptr[5] + 3       # row 4: four columns (valid); row 5: length -2
    row_ptr[R] = 1 << 30              # row R-1: far more than nb columns
    import block_sparse_attention_sba_b200 as sba
    sa, status = _attn_with_csr(wl, q, k, v, row_ptr, col_idx, sched=sched, work_counts=good_counts)
    assert status == sba.SBA_ERR_DEVICE_CHECK
    ot = sa.ot.cpu()
    for r in (5, R - 1):
        b, h, i = r // (wl.H * g.nb), (r // g.nb) % wl.H, r % g.nb
        assert torch.all(ot[b, h, i * g.bs:(i + 1) * g.bs] == 0)
    # a good row computed in the same launch matches the oracle
    qt, kt, vt = (to64(x.cpu()) for x in (sa.qt, sa.kt, sa.vt))
    rp_ok = np.arange(R + 1)
    Ot, _ = oracle.attention(qt, kt, vt, g, rp_ok, col_idx, blocks=[(0, 0, 2)])
    valid = oracle.slot_valid(g)
    sl = slice(2 * g.bs, 3 * g.bs)
    mx, rel = attention_errors(to64(ot)[0, 0, sl][valid[sl]], Ot[0, 0, sl][valid[sl]])
    assert mx <= ATOL and rel <= REL_L2
    _, status2 = _attn_with_csr(wl, q, k, v, rp_ok, col_idx, sched=sched)
    assert status2 == 0


def test_bounded_wait_gives_up_and_reports_timeout():
    """Failure detection without a hang: a wait on a barrier nothing arrives at
    gives up after 2 ms, the status word says so and the context stays usable."""
    _cuda()
    import block_sparse_attention_sba_b200 as sba
    plan = sba.Plan(1, 2, 4, 8, 8, 64, (4, 4, 4), "bf16")
    ws = torch.zeros(plan.info.workspace_bytes, dtype=torch.uint8, device="cuda")
    sba.sba_debug_timeout_probe(plan.handle, ws, 2_000_000)
    assert sba.sba_check_device_status(plan.handle, ws) == sba.SBA_ERR_DEVICE_TIMEOUT
    assert sba.sba_check_device_status(plan.handle, ws) == 0  # cleared
    x = torch.ones(1024, device="cuda")
    assert float((x * 2).sum()) == 2048.0


# ----------------------------------------------------------------- full size

FULL = ["wan", "hunyuan", "stress", "wan_hilbert"]


@pytest.fixture(scope="module", params=FULL)
def full_case(request):
    name = request.param
    wl = (datagen.with_order(datagen.WORKLOADS["wan"], "hilbert") if name == "wan_hilbert"
          else datagen.WORKLOADS[name])
    q, k, v = datagen.generate(wl, seed=0, device=_cuda())
    gpu = run_gpu(wl, q, k, v, with_trace=True)
    return name, wl, (q, k, v), gpu


def test_full_reorder_bit_exact(full_case):
    name, wl, (q, k, v), gpu = full_case
    g = geom_of(wl)
    for h in range(wl.H):
        for x, xt in ((q, gpu["qt"]), (k, gpu["kt"]), (v, gpu["vt"])):
            assert np.array_equal(to64(xt[:, h:h + 1]), oracle.reorder(to64(x[:, h:h + 1].cpu()), g))
        assert np.array_equal(to64(gpu["o"][:, h:h + 1]), oracle.unreorder(to64(gpu["ot"][:, h:h + 1]), g))


def test_full_mask_matches_oracle(full_case):
    name, wl, _, gpu = full_case
    g = geom_of(wl)
    orc = oracle_mask_per_head(wl, to64(gpu["qt"]), to64(gpu["kt"]), wl.top_p_per_head(), wl.top_k)
    stats = compare_mask(gpu, orc, wl.top_p_per_head(), wl.top_k, g.nb, wl.H)
    print(name, stats)
    assert gpu["status"] == 0


def test_full_attention_sampled_blocks(full_case):
    name, wl, _, gpu = full_case
    blocks = sample_blocks(wl, gpu["row_cnt"], per_head=2)
    R, G, lr, lg = oracle_attention_blocks(wl, gpu, blocks)
    mx, rel = attention_errors(G, R)
    print(name, "sampled blocks", len(blocks), "max-abs", mx, "rel-L2", rel)
    assert mx <= ATOL and rel <= REL_L2
    assert np.abs(lr - lg).max() <= 1e-2


def test_full_schedules_agree_and_trace_is_complete(full_case):
    name, wl, (q, k, v), gpu = full_case
    hm = run_gpu(wl, q, k, v, sched=1, with_trace=True)
    assert torch.equal(hm["ot"], gpu["ot"])
    for tr in (gpu["trace"], hm["trace"]):
        assert np.all(tr[:, 1] >= tr[:, 0]) and np.all(tr[:, 0] > 0)
