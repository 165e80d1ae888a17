"""GPU parity of the low-bit P.V path (VC-Attention: Value Smoothing and
Softmax Casting for Low-bit Attention, abstract: V-Smooth, ExpCast-FP8)
through the C ABI.

sba_smooth_v is integer work once its fp32 inputs are fixed: codes, block
means and exponents are compared bit-exactly with the oracle on the GPU's own
reordered values. sba_attention_lowbit is compared with the oracle's low-bit attention on the
GPU's CSR and codes: rel-L2 <= 1e-2 as for bf16, and every output within 2e-2
(lse within 1e-2) plus the oracle's own bound on what codes near a rounding
boundary can change. The kernel rounds 8x + 104 from fp32 tensor-core scores,
the oracle from fp64 scores; a code whose argument lies within rounding
distance of k + 1/2 may come out as the neighbouring code, and the oracle
reports, per query row, how far O and lse can move if all such codes flip. A
query row with a reference-replacement decision within rounding distance of
its threshold is checked against the oracle run that takes that decision the
other way as well (either must match); a row with two such decisions is
exempt and counted. The departure from exact attention is the quantisation
error of the method and is only bounded loosely (rel-L2 < 6 %).
"""
import math

import numpy as np
import pytest
import torch

import datagen
import oracle
from parity_utils import ATOL, REL_L2, attention_errors, geom_of, sample_blocks, to64

pytestmark = pytest.mark.gpu

SMALL = datagen.custom("lowbit_small", 1, 3, 5, 20, 19, 128, (2, 8, 8), top_p=(0.8, 0.9, 0.95),
                       top_k=3, rope_split=(44, 42, 42))


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(wl, seed=0):
    import block_sparse_attention_sba_b200 as sba
    dev = torch.device("cuda:0")
    q, k, v = datagen.generate(wl, seed=seed, device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube, order=getattr(wl, "order", "cube"))
    sa = sba.SparseAttention(plan, device=dev)
    o = sa.lowbit(q, k, v, wl.top_p_per_head(), wl.top_k)
    torch.cuda.synchronize()
    status = sa.check()
    nnz = int(sa.row_ptr[-1].item())
    return {"status": status, "sa": sa, "o": o.cpu(), "qt": sa.qt.cpu(), "kt": sa.kt.cpu(),
            "vt": sa.vt.cpu(), "ot": sa.ot.cpu(), "lse": sa.lse.cpu(),
            "vq": sa.vq.cpu().numpy(), "vmean": sa.vmean.cpu().numpy(),
            "vexp": sa.vexp.cpu().numpy().astype(np.int64),
            "row_cnt": sa.row_cnt.cpu().numpy().astype(np.int64),
            "row_ptr": sa.row_ptr.cpu().numpy().astype(np.int64),
            "col_idx": sa.col_idx[:nnz].cpu().numpy().astype(np.int64)}


def _check_smooth(wl, gpu):
    g = geom_of(wl)
    codes, mu, e = oracle.v_smooth(to64(gpu["vt"]), g)
    B, H = codes.shape[:2]
    ref_q = codes.reshape(B, H, g.nb, g.bs, -1).transpose(0, 1, 2, 4, 3)  # [.., d, bs]
    assert np.array_equal(gpu["vexp"], e)
    assert np.array_equal(gpu["vmean"], mu)
    assert np.array_equal(gpu["vq"], ref_q)
    return codes, mu, e


def _check_attention(wl, gpu, codes, mu, e, blocks):
    g = geom_of(wl)
    valid = oracle.slot_valid(g)
    ref_rows, got_rows, ref_l, got_l, ex_rows, fo_rows, fl_rows = [], [], [], [], [], [], []
    by_head = {}
    for (b, h, i) in blocks:
        by_head.setdefault((b, h), []).append(i)
    n_thr = n_exempt = n_flip_rows = 0
    for (b, h), idx in by_head.items():
        base = (b * wl.H + h) * g.nb
        rp = gpu["row_ptr"][base:base + g.nb + 1] - gpu["row_ptr"][base]
        ci = gpu["col_idx"][gpu["row_ptr"][base]:gpu["row_ptr"][base + g.nb]]
        qt = to64(gpu["qt"][b:b + 1, h:h + 1])
        kt = to64(gpu["kt"][b:b + 1, h:h + 1])
        args = (qt, kt, codes[b:b + 1, h:h + 1], mu[b:b + 1, h:h + 1], e[b:b + 1, h:h + 1], g, rp, ci)
        Ot, lse, dg = oracle.attention_fp8(*args, blocks=[(0, 0, i) for i in idx], diag=True)
        Ox, _ = oracle.attention(qt, kt, to64(gpu["vt"][b:b + 1, h:h + 1]), g, rp, ci,
                                 blocks=[(0, 0, i) for i in idx])
        for i in idx:
            sl = slice(i * g.bs, (i + 1) * g.bs)
            m = valid[sl].copy()
            got_o = to64(gpu["ot"][b, h, sl])
            got_lse = gpu["lse"][b, h, sl].double().numpy()
            o_ref, l_ref = Ot[0, 0, sl].copy(), lse[0, 0, sl].copy()
            fo, fl = dg["flip_o"][0, 0, sl], dg["flip_lse"][0, 0, sl]
            near = dg["thr_near"][0, 0, sl]
            n_thr += int((near[m] > 0).sum())
            n_flip_rows += int((fo.max(axis=1)[m] > 0).sum())
            one = m & (near == 1)
            if one.any():
                # the other decision at the flagged block, for those query rows
                inv = np.zeros((rp[i + 1] - rp[i], g.bs), dtype=bool)
                inv[dg["thr_first"][0, 0, sl][one], np.nonzero(one)[0]] = True
                Oa, la, dga = oracle.attention_fp8(*args, blocks=[(0, 0, i)], invert={(0, 0, i): inv},
                                                   diag=True)
                for q in np.nonzero(one)[0]:
                    fits = lambda o, l, f, fl_: (np.all(np.abs(got_o[q] - o) <= ATOL + f) and
                                                 abs(got_lse[q] - l) <= 1e-2 + fl_)
                    if not fits(o_ref[q], l_ref[q], fo[q], fl[q]):
                        o_ref[q], l_ref[q] = Oa[0, 0, sl][q], la[0, 0, sl][q]
                        fo[q], fl[q] = dga["flip_o"][0, 0, sl][q], dga["flip_lse"][0, 0, sl][q]
            two = m & (near >= 2)
            n_exempt += int(two.sum())
            m &= ~two
            ref_rows.append(o_ref[m])
            ex_rows.append(Ox[0, 0, sl][m])
            got_rows.append(got_o[m])
            ref_l.append(l_ref[m])
            got_l.append(got_lse[m])
            fo_rows.append(fo[m])
            fl_rows.append(fl[m])
    R, G, X = np.concatenate(ref_rows), np.concatenate(got_rows), np.concatenate(ex_rows)
    FO, FL = np.concatenate(fo_rows), np.concatenate(fl_rows)
    mx, rel = attention_errors(G, R)
    err = np.abs(G - R)
    worst = np.unravel_index(int(np.argmax(err - FO)), err.shape)
    info = (mx, rel, worst, float(err[worst]), float(FO[worst]))
    beyond = int((err > ATOL).sum())
    print(f"query rows {R.shape[0]}: with near-boundary codes {n_flip_rows}, near-threshold "
          f"{n_thr}, exempt {n_exempt}; max |err| {mx:.3g}, outputs beyond {ATOL} {beyond} "
          f"(of {err.size}), median flip bound {float(np.median(FO)):.2g}")
    assert rel <= REL_L2, info
    assert np.all(err <= ATOL + FO), info
    dl = np.abs(np.concatenate(got_l) - np.concatenate(ref_l))
    assert np.all(dl <= 1e-2 + FL), (dl.max(),)
    assert n_exempt <= max(2, R.shape[0] // 1000), n_exempt
    _, rel_exact = attention_errors(G, X)
    assert rel_exact < 0.06, rel_exact
    return mx, rel, rel_exact


def test_lowbit_small_every_row():
    _need_gpu()
    gpu = _run(SMALL)
    assert gpu["status"] == 0
    codes, mu, e = _check_smooth(SMALL, gpu)
    g = geom_of(SMALL)
    blocks = [(0, h, i) for h in range(SMALL.H) for i in range(g.nb)]
    _check_attention(SMALL, gpu, codes, mu, e, blocks)


def test_lowbit_wan_layer_sampled_rows():
    """The Wan-shaped layer (40 heads x 308 blocks): smoothing bit-exact on
    every head, attention on sampled rows of every fourth head."""
    _need_gpu()
    wl = datagen.WORKLOADS["wan"]
    gpu = _run(wl)
    assert gpu["status"] == 0
    codes, mu, e = _check_smooth(wl, gpu)
    blocks = [x for x in sample_blocks(wl, gpu["row_cnt"], per_head=1, seed=5) if x[1] % 4 == 0]
    _check_attention(wl, gpu, codes, mu, e, blocks)


def test_lowbit_empty_rows_and_rejected_shapes():
    _need_gpu()
    import block_sparse_attention_sba_b200 as sba
    wl = SMALL
    g = geom_of(wl)
    dev = torch.device("cuda:0")
    q, k, v = datagen.generate(wl, seed=1, device=dev)
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube)
    sa = sba.SparseAttention(plan, device=dev)
    h = plan.handle
    sba.sba_reorder(h, q, k, v, sa.qt, sa.kt, sa.vt, sa.workspace)
    # a stripe mask whose third head keeps nothing: those rows must come out empty
    sba.sba_build_stripe_mask(h, [(3, -1, 0, 5, -2, 0), (1, 0, 0, 1, 0, 0), (1, 9, 0, 1, 0, 0)],
                              sa.bitmask, sa.row_cnt, sa.row_ptr, sa.col_idx, sa.work_order,
                              sa.workspace)
    vq = torch.empty(1, wl.H, g.nb, wl.d, g.bs, dtype=torch.uint8, device=dev)
    vmean = torch.empty(1, wl.H, g.nb, wl.d, dtype=torch.float32, device=dev)
    vexp = torch.empty(1, wl.H, dtype=torch.int32, device=dev)
    sba.sba_smooth_v(h, sa.vt, vq, vmean, vexp, sa.workspace)
    sba.sba_attention_lowbit(h, sa.qt, sa.kt, vq, vmean, vexp, sa.row_ptr, sa.col_idx,
                             sa.work_order, sa.ot, sa.lse, None, sa.workspace)
    torch.cuda.synchronize()
    assert sa.check() == 0
    valid = oracle.slot_valid(g)
    ot = sa.ot.cpu()
    lse = sa.lse.cpu().double().numpy()
    assert torch.all(ot[0, 2] == 0)
    assert np.all(np.isneginf(lse[0, 2][valid]))
    assert torch.isfinite(ot[0, :2].float()).all()
    plan64 = sba.Plan(1, 2, 8, 16, 16, 64, (4, 4, 4), "bf16")
    with pytest.raises(sba.SbaError) as err:
        sba.sba_attention_lowbit(plan64.handle, sa.qt, sa.kt, vq, vmean, vexp, sa.row_ptr,
                                 sa.col_idx, sa.work_order, sa.ot, sa.lse, None, sa.workspace)
    assert err.value.status == sba.SBA_ERR_UNSUPPORTED


def test_lowbit_hilbert_order_every_row():
    """Hilbert-ordered blocks (a partial last block): smoothing counts only the
    real tokens of the tail block, attention masks its padding keys."""
    _need_gpu()
    wl = datagen.with_order(SMALL, "hilbert")
    gpu = _run(wl)
    assert gpu["status"] == 0
    codes, mu, e = _check_smooth(wl, gpu)
    g = geom_of(wl)
    assert g.N % g.bs != 0  # the last block is partial
    blocks = [(0, h, i) for h in range(wl.H) for i in range(g.nb)]
    _check_attention(wl, gpu, codes, mu, e, blocks)


@pytest.mark.parametrize("d,cube", [(64, (4, 4, 4)), (128, (4, 4, 4)), (64, (2, 8, 8))])
def test_smooth_v_other_shapes_and_special_values(d, cube):
    """sba_smooth_v on its own for the head and block sizes other than 128 x
    128 (each takes its own thread mapping), bit-exact against the oracle,
    on ragged grids with: a head whose values are all equal (every residual
    0, so e = 0 and every code 0), and a head holding zeros, negative zeros,
    bf16 subnormals and a few large values. A second call gives the same
    bits (the kernel's counters reset themselves)."""
    _need_gpu()
    import block_sparse_attention_sba_b200 as sba
    dev = torch.device("cuda:0")
    B, H, T, Hh, W = 1, 3, 5, 9, 11
    N = T * Hh * W
    _, _, v = datagen.random_qkv(B, H, N, d, seed=7)
    v = v.clone()
    v[0, 1] = 0.375
    rng = np.random.default_rng(11)
    flat = v[0, 2].view(-1)
    for val, n in ((0.0, 200), (-0.0, 200), (1e-40, 50), (-3e-39, 50), (300.0, 3)):
        idx = torch.from_numpy(rng.choice(flat.numel(), n, replace=False))
        flat[idx] = torch.tensor(val, dtype=torch.bfloat16)
    v = v.to(dev)
    plan = sba.Plan(B, H, T, Hh, W, d, cube, "bf16")
    sa = sba.SparseAttention(plan, device=dev)
    inf = plan.info
    h = plan.handle
    sba.sba_reorder(h, v, v, v, sa.qt, sa.kt, sa.vt, sa.workspace)
    g = oracle.Geom(T, Hh, W, *cube)
    codes, mu, e = oracle.v_smooth(to64(sa.vt.cpu()), g)
    ref_q = codes.reshape(B, H, g.nb, g.bs, d).transpose(0, 1, 2, 4, 3)
    assert e[0, 1] == 0 and not ref_q[0, 1].any()
    assert e[0, 2] > e[0, 0]  # the large values set head 2's scale
    for _ in range(2):
        vq = torch.full((B, H, inf.nb, d, inf.bs), 0xAB, dtype=torch.uint8, device=dev)
        vmean = torch.full((B, H, inf.nb, d), float("nan"), dtype=torch.float32, device=dev)
        vexp = torch.full((B, H), -999, dtype=torch.int32, device=dev)
        sba.sba_smooth_v(h, sa.vt, vq, vmean, vexp, sa.workspace)
        torch.cuda.synchronize()
        assert sa.check() == 0
        assert np.array_equal(vexp.cpu().numpy().astype(np.int64), e)
        assert np.array_equal(vmean.cpu().numpy(), mu)
        assert np.array_equal(vq.cpu().numpy(), ref_q)
