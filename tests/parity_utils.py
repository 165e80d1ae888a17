"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same bits, and compare the way the acceptance rules say.

Attention tolerance (bf16 operands, fp32 accumulation): max-abs <= 2e-2 and
relative L2 <= 1e-2 over the real query slots. Permutation, CSR indexing and
work order: bit-exact. Mask rows: identical to the oracle except rows whose
cumulative mass at the cut lies within 1e-4 of p (boundary); those rows are
counted and must still satisfy the routing invariants. No other exemption:
the library routes in fp64 like the oracle.

The library takes Top-p values as fp32; the oracle is given the same fp32
values (widened to fp64), so both cut at the same p.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from oracle import Geom

ATOL = 2e-2
REL_L2 = 1e-2
BOUNDARY_TOL = 1e-4


def as_fp32(top_p):
    """The Top-p values as the library receives them (fp32), widened back."""
    return [float(np.float32(x)) for x in top_p]


def geom_of(wl) -> Geom:
    return Geom(wl.T, wl.Hh, wl.W, *wl.cube, order=getattr(wl, "order", "cube"))


def run_gpu(wl, q, k, v, sched=0, with_trace=False, top_p=None, top_k=None):
    """All four calls on cuda:0; returns a dict of CPU tensors."""
    import block_sparse_attention_sba_b200 as sba
    plan = sba.Plan.for_tensor(q, wl.T, wl.Hh, wl.W, wl.cube, order=getattr(wl, "order", "cube"))
    sa = sba.SparseAttention(plan, device=q.device)
    top_p = wl.top_p_per_head() if top_p is None else top_p
    top_k = wl.top_k if top_k is None else top_k
    trace = None
    if with_trace:
        trace = torch.zeros(plan.info.rows * 3, dtype=torch.int64, device=q.device)
    o = sa(q, k, v, top_p, top_k, sched=sched, trace=trace)
    torch.cuda.synchronize()
    status = sa.check()
    nnz = int(sa.row_ptr[-1].item())
    out = {
        "plan": plan, "status": status,
        "qt": sa.qt.cpu(), "kt": sa.kt.cpu(), "vt": sa.vt.cpu(), "ot": sa.ot.cpu(),
        "o": o.cpu(), "lse": sa.lse.cpu(),
        "row_cnt": sa.row_cnt.cpu().numpy().astype(np.int64),
        "row_ptr": sa.row_ptr.cpu().numpy().astype(np.int64),
        "col_idx": sa.col_idx[:nnz].cpu().numpy().astype(np.int64),
        "bitmask": sa.bitmask.cpu().numpy().view(np.uint32),
        "work_order": sa.work_order.cpu().numpy().astype(np.int64),
    }
    if with_trace:
        out["trace"] = trace.cpu().numpy().reshape(-1, 3)
    return out


def to64(x: torch.Tensor) -> np.ndarray:
    return x.double().numpy()


def oracle_mask_per_head(wl, qt: np.ndarray, kt: np.ndarray, top_p, top_k):
    """Oracle routing head by head (bounded memory); rows concatenated in
    (b, h, i) order."""
    g = geom_of(wl)
    top_p = as_fp32(top_p)
    parts = []
    for b in range(qt.shape[0]):
        for h in range(qt.shape[1]):
            parts.append(oracle.build_mask(qt[b:b + 1, h:h + 1], kt[b:b + 1, h:h + 1], g,
                                           [top_p[h]], top_k, BOUNDARY_TOL))
    keys = ["row_cnt", "boundary"]
    res = {k: np.concatenate([p[k] for p in parts]) for k in keys}
    res["bitmask"] = np.concatenate([p["bitmask"] for p in parts])
    res["probs"] = np.concatenate([p["probs"].reshape(-1, g.nb) for p in parts])
    res["cols"] = [p["col_idx"][p["row_ptr"][i]:p["row_ptr"][i + 1]]
                   for p in parts for i in range(g.nb)]
    return res


def compare_mask(gpu: dict, orc: dict, top_p, top_k: int, nb: int, H: int) -> dict:
    """Bit-exact CSR bookkeeping; per-row equality except boundary rows."""
    top_p = as_fp32(top_p)
    R = gpu["row_cnt"].size
    rc = gpu["row_cnt"]
    assert gpu["row_ptr"][0] == 0
    assert np.array_equal(gpu["row_ptr"][1:], np.cumsum(rc)), "row_ptr is not the scan of row_cnt"
    assert np.array_equal(gpu["work_order"], oracle.lpt_order(rc, nb)), "work order differs"
    words = (nb + 31) // 32
    mism = boundary = 0
    for r in range(R):
        cols = gpu["col_idx"][gpu["row_ptr"][r]:gpu["row_ptr"][r + 1]]
        assert np.all(np.diff(cols) > 0) and (cols.size == 0 or (cols[0] >= 0 and cols[-1] < nb))
        flags = np.zeros(words * 32, dtype=bool)
        flags[cols] = True
        bits = np.packbits(flags, bitorder="little").view("<u4")
        assert np.array_equal(bits, gpu["bitmask"][r]), f"row {r}: bitmask != CSR"
        if np.array_equal(cols, orc["cols"][r]):
            continue
        mism += 1
        if orc["boundary"][r]:
            boundary += 1
        else:
            raise AssertionError(
                f"row {r}: mask differs from the oracle outside the exemptions "
                f"(gpu {cols.tolist()[:12]}.. n={cols.size}, oracle n={orc['cols'][r].size})")
        p = top_p[(r // nb) % H]
        P = orc["probs"][r]
        assert cols.size >= min(top_k, nb)
        assert P[cols].sum() >= p - BOUNDARY_TOL or cols.size == nb
    return {"rows": R, "mismatch": mism, "boundary_exempt": boundary,
            "boundary_rows_oracle": int(orc["boundary"].sum()),
            "density": float(rc.sum()) / (R * nb)}


def attention_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    d = o_gpu - o_ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-30))


def sample_blocks(wl, row_cnt: np.ndarray, per_head: int = 4, seed: int = 0):
    """Query blocks the oracle recomputes at full size: per head the last
    (edge) block, the heaviest and lightest rows, and random others."""
    g = geom_of(wl)
    rng = np.random.default_rng(seed)
    out = []
    for b in range(wl.B):
        for h in range(wl.H):
            base = (b * wl.H + h) * g.nb
            cnt = row_cnt[base:base + g.nb]
            pick = {g.nb - 1, int(np.argmax(cnt)), int(np.argmin(cnt))}
            while len(pick) < per_head + 3:
                pick.add(int(rng.integers(0, g.nb)))
            out += [(b, h, i) for i in sorted(pick)]
    return out


def oracle_attention_blocks(wl, gpu: dict, blocks):
    """Oracle attention for the chosen blocks on the GPU's own CSR (so the
    attention check is independent of mask exemptions). Returns per-block
    (valid rows of O, lse) pairs and the GPU's."""
    g = geom_of(wl)
    valid = oracle.slot_valid(g)
    errs = []
    ref_rows, gpu_rows, ref_lse, gpu_lse = [], [], [], []
    by_head = {}
    for (b, h, i) in blocks:
        by_head.setdefault((b, h), []).append(i)
    for (b, h), idx in by_head.items():
        qt = to64(gpu["qt"][b:b + 1, h:h + 1])
        kt = to64(gpu["kt"][b:b + 1, h:h + 1])
        vt = to64(gpu["vt"][b:b + 1, h:h + 1])
        base = (b * wl.H + h) * g.nb
        rp = gpu["row_ptr"][base:base + g.nb + 1] - gpu["row_ptr"][base]
        ci = gpu["col_idx"][gpu["row_ptr"][base]:gpu["row_ptr"][base + g.nb]]
        Ot, lse = oracle.attention(qt, kt, vt, g, rp, ci, blocks=[(0, 0, i) for i in idx])
        for i in idx:
            sl = slice(i * g.bs, (i + 1) * g.bs)
            m = valid[sl]
            ref_rows.append(Ot[0, 0, sl][m])
            gpu_rows.append(to64(gpu["ot"][b, h, sl])[m])
            ref_lse.append(lse[0, 0, sl][m])
            gpu_lse.append(gpu["lse"][b, h, sl].double().numpy()[m])
            assert np.all(to64(gpu["ot"][b, h, sl])[~m] == 0), "padding query rows must be zero"
    R = np.concatenate(ref_rows)
    G = np.concatenate(gpu_rows)
    return R, G, np.concatenate(ref_lse), np.concatenate(gpu_lse)
