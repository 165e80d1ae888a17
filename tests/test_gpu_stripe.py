"""GPU parity of the stripe mask (Parameterized Stripe Attention for Efficient
Video Generation, Approach: M(Tw, To, Ts, Sw, So, Ss)) through the C ABI.

Bitmask, row_cnt, row_ptr, col_idx and the work order are integer work:
bit-exact against the oracle. Attention over the stripe CSR: within the bf16
tolerance of the other parity tests (max-abs <= 2e-2, relative L2 <= 1e-2;
lse within 1e-2); rows the stripes leave empty give zero output and
lse = -inf on real query slots."""
import numpy as np
import pytest
import torch

import datagen
import oracle
from parity_utils import (ATOL, REL_L2, attention_errors, geom_of, oracle_attention_blocks,
                          sample_blocks, to64)

pytestmark = pytest.mark.gpu


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(wl, params, sched=0, seed=0):
    import block_sparse_attention_sba_b200 as sba
    dev = torch.device("cuda:0")
    q, k, v = datagen.generate(wl, seed=seed, device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube)
    sa = sba.SparseAttention(plan, device=dev)
    o = sa.stripe(q, k, v, params, sched=sched)
    torch.cuda.synchronize()
    status = sa.check()
    nnz = int(sa.row_ptr[-1].item())
    return {
        "status": status, "qt": sa.qt.cpu(), "kt": sa.kt.cpu(), "vt": sa.vt.cpu(),
        "ot": sa.ot.cpu(), "o": o.cpu(), "lse": sa.lse.cpu(),
        "row_cnt": sa.row_cnt.cpu().numpy().astype(np.int64),
        "row_ptr": sa.row_ptr.cpu().numpy().astype(np.int64),
        "col_idx": sa.col_idx[:nnz].cpu().numpy().astype(np.int64),
        "bitmask": sa.bitmask.cpu().numpy().view(np.uint32),
        "work_order": sa.work_order.cpu().numpy().astype(np.int64),
    }


def _check_csr(wl, params, gpu):
    g = geom_of(wl)
    ref = oracle.stripe_mask(g, params, wl.B)
    for key in ("row_cnt", "row_ptr", "col_idx", "bitmask"):
        assert np.array_equal(gpu[key], np.asarray(ref[key]).astype(gpu[key].dtype)), key
    assert np.array_equal(gpu["work_order"], oracle.lpt_order(ref["row_cnt"], g.nb))
    return ref


def _check_attention(wl, gpu, blocks):
    g = geom_of(wl)
    valid = oracle.slot_valid(g)
    cnt = gpu["row_cnt"]
    row = lambda b, h, i: (b * wl.H + h) * g.nb + i
    nonempty = [x for x in blocks if cnt[row(*x)] > 0]
    empty = [x for x in blocks if cnt[row(*x)] == 0]
    if nonempty:
        R, G, lr, lg = oracle_attention_blocks(wl, gpu, nonempty)
        mx, rel = attention_errors(G, R)
        assert mx <= ATOL and rel <= REL_L2, (mx, rel)
        assert np.abs(lg - lr).max() <= 1e-2
    for (b, h, i) in empty:
        sl = slice(i * g.bs, (i + 1) * g.bs)
        assert np.all(to64(gpu["ot"][b, h, sl]) == 0)
        assert np.all(np.isneginf(gpu["lse"][b, h, sl].double().numpy()[valid[sl]]))
    return len(nonempty), len(empty)


SMALL = {
    # nT x nH x nW = 3 x 3 x 3 with ragged edges; head 2's stripes miss the grid
    "ragged_d128": (datagen.custom("stripe_ragged_d128", 1, 3, 5, 20, 19, 128, (2, 8, 8),
                                   top_p=(1.0,) * 3, top_k=0, rope_split=(44, 42, 42)),
                    [(3, -1, 0, 5, -2, 0), (1, 0, 2, 3, -1, 3), (1, 9, 0, 1, 0, 0)]),
    # bs = 64, d = 64, two batches, nb = 32 (one full bitmask word)
    "d64_bs64": (datagen.custom("stripe_d64_bs64", 2, 2, 8, 16, 16, 64, (4, 4, 4),
                                top_p=(1.0,) * 2, top_k=0, rope_split=(22, 22, 20)),
                 [(2, -1, 0, 7, -3, 4), (3, -1, 0, 9, -4, 0)]),
    # fp32 path
    "f32": (datagen.custom("stripe_f32", 1, 2, 5, 6, 7, 64, (4, 4, 4), dtype="f32",
                           top_p=(1.0,) * 2, top_k=0, rope_split=(22, 22, 20)),
            [(1, 0, 0, 1, 0, 0), (2, -1, 0, 3, -1, 2)]),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("sched", [0, 1])
def test_stripe_small_all_rows(name, sched):
    _need_gpu()
    wl, params = SMALL[name]
    gpu = _run(wl, params, sched=sched)
    assert gpu["status"] == 0
    _check_csr(wl, params, gpu)
    g = geom_of(wl)
    blocks = [(b, h, i) for b in range(wl.B) for h in range(wl.H) for i in range(g.nb)]
    n_ok, n_empty = _check_attention(wl, gpu, blocks)
    assert n_ok > 0
    if name == "ragged_d128":
        assert n_empty == g.nb  # head 2
        # the raster output is the oracle's unreorder of the cube-ordered one
        assert torch.equal(gpu["o"], torch.from_numpy(
            oracle.unreorder(gpu["ot"].float().numpy(), g)).to(gpu["o"].dtype))


def test_stripe_full_size_wan_geometry():
    """A Wan-shaped layer (40 heads, 308 blocks of 128 tokens): every head has
    its own stripes; CSR bit-exact, attention on sampled rows of every fourth
    head."""
    _need_gpu()
    wl = datagen.WORKLOADS["wan"]
    g = geom_of(wl)
    nS = g.nH * g.nW
    pats = [(5, -2, 0, 2 * g.nW + 3, -(g.nW + 1), 0),   # local window
            (3, -1, 0, 3, -1, g.nW),                     # column stripes every cube row
            (1, 0, 2, nS, 0, 0),                         # even frame offsets, one frame row
            (2 * g.nT - 1, -(g.nT - 1), 0, 1, 0, 0)]     # same spatial cube, all frames
    params = [pats[h % len(pats)] for h in range(wl.H)]
    gpu = _run(wl, params)
    assert gpu["status"] == 0
    _check_csr(wl, params, gpu)
    blocks = [x for x in sample_blocks(wl, gpu["row_cnt"], per_head=1, seed=2) if x[1] % 4 == 0]
    n_ok, _ = _check_attention(wl, gpu, blocks)
    assert n_ok > 0
