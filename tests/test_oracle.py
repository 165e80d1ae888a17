"""Pins for the fp64 oracle against things other than itself: hand-worked
examples, brute force over tiny inputs, closed forms, library routines and
invariants. CPU only.

Each group names the plausible mistake it is there to catch.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle import Geom

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

GEOMS = [
    Geom(4, 8, 8, 4, 4, 4),      # tiny workload grid (divisible)
    Geom(8, 16, 16, 4, 4, 4),    # small workload grid (divisible)
    Geom(5, 9, 7, 2, 4, 4),      # ragged in every axis
    Geom(3, 3, 3, 2, 2, 2),
    Geom(1, 1, 1, 1, 1, 1),
    Geom(2, 3, 3, 1, 2, 2),
    Geom(21, 30, 52, 2, 8, 8),   # Wan-shaped grid (ragged t, h, w)
]


# ----------------------------------------------------------------- permutation
# catches: swapped axes, wrong cube-grid strides, wrong in-cube order

@pytest.mark.parametrize("g", GEOMS, ids=str)
def test_perm_formula_matches_explicit_loops(g):
    assert np.array_equal(oracle.slot_of_token(g), oracle.slot_of_token_loops(g))


def test_perm_hand_worked_example():
    lines = [l for l in open(os.path.join(GOLDEN, "perm_worked.txt")) if not l.startswith("#")]
    kv = {l.split(":")[0]: [int(x) for x in l.split(":")[1].split()] for l in lines if ":" in l}
    g = Geom(*kv["geometry"])
    assert oracle.slot_of_token(g).tolist() == kv["slot_of_token"]
    assert oracle.block_len(g).tolist() == kv["block_len"]


@pytest.mark.parametrize("g", [Geom(4, 8, 8, 4, 4, 4), Geom(8, 16, 16, 4, 4, 4),
                               Geom(4, 16, 24, 2, 8, 8)], ids=str)
def test_perm_divisible_grid_is_a_6d_transpose(g):
    """With no padding the cube order is the textbook reshape/transpose."""
    rng = np.random.default_rng(1)
    d = 3
    X = rng.standard_normal((1, 1, g.N, d))
    ref = (X.reshape(g.nT, g.ct, g.nH, g.ch, g.nW, g.cw, d)
           .transpose(0, 2, 4, 1, 3, 5, 6).reshape(1, 1, g.Npad, d))
    assert np.array_equal(oracle.reorder(X, g), ref)


@pytest.mark.parametrize("g", GEOMS, ids=str)
def test_perm_is_injective_onto_valid_slots_and_cubes_are_boxes(g):
    s = oracle.slot_of_token(g)
    assert np.unique(s).size == g.N and s.min() >= 0 and s.max() < g.Npad
    valid = oracle.slot_valid(g)
    assert valid.sum() == g.N and np.array_equal(np.nonzero(valid)[0], np.sort(s))
    t, h, w = np.unravel_index(np.arange(g.N), (g.T, g.Hh, g.W))
    blk = s // g.bs
    for b in np.unique(blk):
        m = blk == b
        for c, e in ((t[m], g.ct), (h[m], g.ch), (w[m], g.cw)):
            assert c.min() // e == c.max() // e  # one aligned box per block
    # the real slots of every block are a prefix of it (padding at the tail)
    V = valid.reshape(g.nb, g.bs)
    for b in range(g.nb):
        n_real = int(V[b].sum())
        assert V[b, :n_real].all() and not V[b, n_real:].any()
    # closed form for block lengths: product of per-axis clipped extents
    L = oracle.block_len(g).reshape(g.nT, g.nH, g.nW)
    for tt, th, tw in itertools.product(range(g.nT), range(g.nH), range(g.nW)):
        exp = (min(g.ct, g.T - tt * g.ct) * min(g.ch, g.Hh - th * g.ch)
               * min(g.cw, g.W - tw * g.cw))
        assert L[tt, th, tw] == exp
    assert L.sum() == g.N


@pytest.mark.parametrize("g", GEOMS[:6], ids=str)
def test_reorder_round_trip_and_zero_padding(g):
    rng = np.random.default_rng(2)
    X = rng.standard_normal((2, 3, g.N, 5))
    Xt = oracle.reorder(X, g)
    assert np.array_equal(oracle.unreorder(Xt, g), X)
    assert np.all(Xt[:, :, ~oracle.slot_valid(g)] == 0)


# --------------------------------------------------------------------- pooling
# catches: dividing by bs instead of the valid count, pooling padding slots

@pytest.mark.parametrize("g", GEOMS[:6], ids=str)
def test_pool_of_blockwise_constant_field_is_that_constant(g):
    rng = np.random.default_rng(3)
    d = 4
    C = rng.standard_normal((1, 2, g.nb, d))
    blk = oracle.slot_of_token(g) // g.bs
    X = C[:, :, blk]  # raster field constant on every cube
    Qbar = oracle.pool(oracle.reorder(X, g), g)
    np.testing.assert_allclose(Qbar, C, rtol=0, atol=1e-12)


def test_pool_matches_explicit_mean_over_tokens():
    g = Geom(5, 9, 7, 2, 4, 4)
    rng = np.random.default_rng(4)
    X = rng.standard_normal((1, 1, g.N, 3))
    blk = oracle.slot_of_token(g) // g.bs
    Qbar = oracle.pool(oracle.reorder(X, g), g)
    for b in range(g.nb):
        np.testing.assert_allclose(Qbar[0, 0, b], X[0, 0, blk == b].mean(axis=0), atol=1e-13)


# --------------------------------------------------------------- block softmax
# catches: wrong 1/sqrt(d) scale, transposed product, missing max shift

def test_block_probs_matches_scipy_softmax():
    rng = np.random.default_rng(5)
    Qb = rng.standard_normal((2, 3, 11, 16)) * 3
    Kb = rng.standard_normal((2, 3, 11, 16)) * 3
    P = oracle.block_probs(Qb, Kb)
    S = np.einsum("bhid,bhjd->bhij", Qb, Kb) / 4.0
    np.testing.assert_allclose(P, scipy.special.softmax(S, axis=-1), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)


def test_block_probs_closed_form_scale():
    d = 9
    a = 2.0
    b = np.array([0.0, 1.0, 3.0, -1.5])
    Qb = np.zeros((1, d)); Qb[0, 0] = a
    Kb = np.zeros((4, d)); Kb[:, 0] = b
    # a single query row against four key rows: exp(a*b_j/3) / sum
    P = oracle.block_probs(Qb, Kb)[0]
    e = np.exp(a * b / 3.0)
    np.testing.assert_allclose(P, e / e.sum(), rtol=1e-14)
    # asymmetric rows: P[i, j] uses Q row i and K row j, not the transpose
    Qb2 = np.stack([Qb[0], 2 * Qb[0]])
    P2 = oracle.block_probs(Qb2, Kb[:2])
    e2 = np.exp(2 * a * b[:2] / 3.0)
    np.testing.assert_allclose(P2[1], e2 / e2.sum(), rtol=1e-14)


def test_block_probs_survive_huge_scores():
    Qb = np.array([[800.0, 0.0]])
    Kb = np.array([[1.0, 0.0], [0.9, 0.0]])
    P = oracle.block_probs(Qb, Kb)
    assert np.all(np.isfinite(P)) and abs(P.sum() - 1) < 1e-12


# ------------------------------------------------------------------- selection
# catches: exclusive instead of inclusive cut, wrong tie order, floor ignored

def _golden_rows():
    for line in open(os.path.join(GOLDEN, "select_worked.txt")):
        if line.startswith("#") or not line.strip():
            continue
        probs, p, k, exp = [x.strip() for x in line.split("|")]
        yield ([float(x) for x in probs.split(",")], float(p), int(k),
               [int(x) for x in exp.split(",")])


@pytest.mark.parametrize("probs,p,k,exp", list(_golden_rows()))
def test_select_hand_worked(probs, p, k, exp):
    sel, _ = oracle.select_row(np.array(probs), p, k)
    assert sel.tolist() == exp


def _brute_force_select(P_frac, p_frac, k):
    """Exact (rational) brute force over every subset: the smallest subset
    size whose best subset reaches mass p, floored at k and capped at nkb;
    among the heaviest subsets of that size the lexicographically smallest
    index tuple (the lower-index tie rule)."""
    nkb = len(P_frac)
    n_p = nkb
    for n in range(1, nkb + 1):
        best = max(sum(P_frac[j] for j in c) for c in itertools.combinations(range(nkb), n))
        if best >= p_frac:
            n_p = n
            break
    n = min(nkb, max(k, n_p))
    cands = list(itertools.combinations(range(nkb), n))
    best = max(sum(P_frac[j] for j in c) for c in cands)
    return min(c for c in cands if sum(P_frac[j] for j in c) == best)


@pytest.mark.parametrize("seed", range(60))
def test_select_matches_brute_force_over_subsets(seed):
    rng = np.random.default_rng(100 + seed)
    nkb = int(rng.integers(1, 10))
    # dyadic probabilities: integers over 64, frequent ties, exact sums
    w = rng.integers(0, 6, size=nkb) if seed % 3 else rng.integers(0, 3, size=nkb)
    if w.sum() == 0:
        w[0] = 1
    denom = 1 << 10
    raw = (w * (denom // w.sum())).astype(np.int64)
    raw[0] += denom - raw.sum()
    if raw[0] < 0:
        return
    P_frac = [Fraction(int(x), denom) for x in raw]
    p_frac = Fraction(int(rng.integers(1, denom + 1)), denom)
    k = int(rng.integers(0, nkb + 2))
    sel, _ = oracle.select_row(np.array([float(x) for x in P_frac]), float(p_frac), k)
    assert tuple(sel.tolist()) == _brute_force_select(P_frac, p_frac, k)


def test_select_special_cases():
    rng = np.random.default_rng(7)
    P = scipy.special.softmax(rng.standard_normal(50) * 2)
    assert oracle.select_row(P, 1.0, 1)[0].size == 50          # p = 1 keeps all
    for k in (1, 3, 7):
        sel, _ = oracle.select_row(P, 1e-12, k)                 # p -> 0: exactly top k
        assert sel.tolist() == sorted(np.argsort(-P, kind="stable")[:k].tolist())
    assert oracle.select_row(P, 0.5, 80)[0].size == 50         # k > nkb caps


def _mask_invariants(m, top_p, top_k, nb):
    R = m["row_cnt"].size
    assert np.array_equal(m["row_ptr"][1:] - m["row_ptr"][:-1], m["row_cnt"])
    assert m["row_ptr"][0] == 0 and np.all(np.diff(m["row_ptr"]) >= 0)
    P = m["probs"].reshape(R, nb)
    H = len(top_p)
    for r in range(R):
        cols = m["col_idx"][m["row_ptr"][r]:m["row_ptr"][r + 1]]
        assert np.all(np.diff(cols) > 0)
        bits = [j for j in range(nb) if (m["bitmask"][r, j // 32] >> (j % 32)) & 1]
        assert bits == cols.tolist()
        p = top_p[(r // nb) % H]
        assert cols.size >= min(top_k, nb)
        mass = P[r, cols].sum()
        assert mass >= p - 1e-12 or cols.size == nb
        if cols.size > max(top_k, 1):          # minimality of the Top-p prefix
            assert mass - P[r, cols].min() < p + 1e-12


def test_build_mask_invariants_ragged():
    g = Geom(5, 9, 7, 2, 4, 4)
    rng = np.random.default_rng(8)
    q = rng.standard_normal((2, 3, g.N, 8)) * 2
    k = rng.standard_normal((2, 3, g.N, 8)) * 2
    top_p = [0.5, 0.8, 0.95]
    m = oracle.build_mask(oracle.reorder(q, g), oracle.reorder(k, g), g, top_p, 2)
    _mask_invariants(m, top_p, 2, g.nb)


def test_lpt_order_matches_python_sort():
    rng = np.random.default_rng(9)
    nb = 20
    cnt = rng.integers(0, 12, size=25 * nb)
    cnt[3 * nb:4 * nb] = cnt[7 * nb:8 * nb]          # two heads with equal totals
    tot = cnt.reshape(25, nb).sum(1)
    exp = sorted(range(cnt.size), key=lambda r: (-tot[r // nb], r // nb, -cnt[r], r))
    assert oracle.lpt_order(cnt, nb).tolist() == exp


def test_lpt_order_single_head_is_plain_longest_first():
    cnt = np.array([3, 7, 7, 1, 0, 7, 2])
    assert oracle.lpt_order(cnt, 7).tolist() == [1, 2, 5, 0, 6, 3, 4]


# ------------------------------------------------------------------- attention
# catches: padding keys not masked, transposed Q/K, wrong scale, padding rows

def _dense_sdpa(qt, kt, vt, g):
    """torch scaled_dot_product_attention in fp64 with a key-padding mask."""
    valid = torch.from_numpy(oracle.slot_valid(g))
    mask = valid[None, None, None, :].expand(qt.shape[0], qt.shape[1], qt.shape[2], -1)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qt), torch.from_numpy(kt), torch.from_numpy(vt), attn_mask=mask).numpy()


@pytest.mark.parametrize("g", [Geom(5, 9, 7, 2, 4, 4), Geom(4, 8, 8, 4, 4, 4)], ids=str)
def test_attention_p1_equals_dense_sdpa(g):
    rng = np.random.default_rng(10)
    q, k, v = (rng.standard_normal((1, 2, g.N, 16)) * s for s in (1.5, 1.5, 1.0))
    qt, kt, vt = (oracle.reorder(x, g) for x in (q, k, v))
    m = oracle.build_mask(qt, kt, g, [1.0, 1.0], 1)
    assert np.all(m["row_cnt"] == g.nb)
    Ot, lse = oracle.attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"])
    ref = _dense_sdpa(qt, kt, vt, g)
    valid = oracle.slot_valid(g)
    np.testing.assert_allclose(Ot[:, :, valid], ref[:, :, valid], atol=1e-12, rtol=1e-10)
    assert np.all(Ot[:, :, ~valid] == 0)
    S = np.einsum("bhqd,bhkd->bhqk", qt, kt) / 4.0
    S[..., ~valid] = -np.inf
    np.testing.assert_allclose(lse[:, :, valid], scipy.special.logsumexp(S, axis=-1)[:, :, valid],
                               atol=1e-12)


def test_attention_closed_form_two_keys():
    # d = 2, q = (sqrt2 ln3, 0), keys e0 and e1: weights 3/4 and 1/4, lse = ln 4
    g = Geom(1, 1, 2, 1, 1, 2)
    qt = np.zeros((1, 1, 2, 2)); qt[0, 0, 0, 0] = math.sqrt(2) * math.log(3)
    kt = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    vt = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    Ot, lse = oracle.attention(qt, kt, vt, g, np.array([0, 1]), np.array([0]))
    np.testing.assert_allclose(Ot[0, 0, 0], [0.75, 0.25], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 0], math.log(4), atol=1e-15)


def test_attention_explicit_loops_on_sparse_mask():
    g = Geom(3, 3, 3, 2, 2, 2)
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((1, 1, g.N, 4)) for _ in range(3))
    qt, kt, vt = (oracle.reorder(x, g) for x in (q, k, v))
    m = oracle.build_mask(qt, kt, g, [0.6], 2)
    assert m["row_cnt"].min() < g.nb  # really sparse
    Ot, lse = oracle.attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"])
    valid = oracle.slot_valid(g)
    for i in range(g.nb):
        sel = m["col_idx"][m["row_ptr"][i]:m["row_ptr"][i + 1]]
        for a in range(i * g.bs, (i + 1) * g.bs):
            if not valid[a]:
                continue
            num = np.zeros(4)
            den = 0.0
            for j in sel:
                for c in range(j * g.bs, (j + 1) * g.bs):
                    if valid[c]:
                        wgt = math.exp(sum(qt[0, 0, a, x] * kt[0, 0, c, x] for x in range(4)) / 2.0)
                        num += wgt * vt[0, 0, c]
                        den += wgt
            np.testing.assert_allclose(Ot[0, 0, a], num / den, atol=1e-12)
            np.testing.assert_allclose(lse[0, 0, a], math.log(den), atol=1e-12)


def test_attention_rows_are_convex_combinations_and_constant_v():
    g = Geom(5, 9, 7, 2, 4, 4)
    rng = np.random.default_rng(12)
    q, k = (rng.standard_normal((1, 2, g.N, 8)) * 2 for _ in range(2))
    v = rng.standard_normal((1, 2, g.N, 8))
    qt, kt, vt = (oracle.reorder(x, g) for x in (q, k, v))
    m = oracle.build_mask(qt, kt, g, [0.7, 0.9], 1)
    Ot, _ = oracle.attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"])
    valid = oracle.slot_valid(g)
    for h in range(2):
        for i in range(g.nb):
            r = h * g.nb + i
            sel = m["col_idx"][m["row_ptr"][r]:m["row_ptr"][r + 1]]
            ks = np.concatenate([np.arange(j * g.bs, (j + 1) * g.bs) for j in sel])
            ks = ks[valid[ks]]
            lo, hi = vt[0, h, ks].min(0), vt[0, h, ks].max(0)
            for a in range(i * g.bs, (i + 1) * g.bs):
                if valid[a]:
                    assert np.all(Ot[0, h, a] >= lo - 1e-12) and np.all(Ot[0, h, a] <= hi + 1e-12)
    vconst = np.broadcast_to(np.arange(8.0), v.shape).copy()
    Oc, _ = oracle.attention(qt, kt, oracle.reorder(vconst, g), g, m["row_ptr"], m["col_idx"])
    np.testing.assert_allclose(Oc[:, :, valid], np.broadcast_to(np.arange(8.0), Oc[:, :, valid].shape),
                               atol=1e-12)


def test_attention_single_valid_key_returns_its_value():
    g = Geom(1, 1, 3, 1, 1, 2)  # block 1 holds one real token (w = 2)
    rng = np.random.default_rng(13)
    qt, kt, vt = (oracle.reorder(rng.standard_normal((1, 1, 3, 4)), g) for _ in range(3))
    Ot, _ = oracle.attention(qt, kt, vt, g, np.array([0, 1, 2]), np.array([1, 1]))
    np.testing.assert_allclose(Ot[0, 0, 0], vt[0, 0, 2], atol=1e-15)
    np.testing.assert_allclose(Ot[0, 0, 2], vt[0, 0, 2], atol=1e-15)


def test_attention_invariant_to_key_order_inside_a_block():
    g = Geom(4, 8, 8, 4, 4, 4)
    rng = np.random.default_rng(14)
    qt, kt, vt = (oracle.reorder(rng.standard_normal((1, 1, g.N, 8)), g) for _ in range(3))
    m = oracle.build_mask(qt, kt, g, [0.8], 1)
    O1, l1 = oracle.attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"])
    perm = np.concatenate([j * g.bs + rng.permutation(g.bs) for j in range(g.nb)])
    O2, l2 = oracle.attention(qt, kt[:, :, perm], vt[:, :, perm], g, m["row_ptr"], m["col_idx"])
    np.testing.assert_allclose(O1, O2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


# ------------------------------------------------------------------ end to end

def test_forward_on_tiny_workload_is_consistent():
    import datagen
    wl = datagen.WORKLOADS["tiny"]
    q, k, v = (x.double().numpy() for x in datagen.generate(wl))
    g = Geom(wl.T, wl.Hh, wl.W, *wl.cube)
    o, m, lse = oracle.forward(q, k, v, g, wl.top_p_per_head(), wl.top_k)
    assert o.shape == q.shape and np.all(np.isfinite(o))
    _mask_invariants(m, wl.top_p_per_head(), wl.top_k, g.nb)


# ------------------------------------------------------------- Hilbert order
# catches: broken reflections / axis swaps (non-adjacent steps), wrong bit
# interleave (sub-cubes not contiguous), rank vs index mix-ups on ragged grids

from oracle.oracle import hilbert_index


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_hilbert_curve_is_a_bijective_unit_step_walk(bits):
    side = 1 << bits
    pts = [(x, y, z) for x in range(side) for y in range(side) for z in range(side)]
    idx = [hilbert_index(*p, bits) for p in pts]
    assert sorted(idx) == list(range(side ** 3))
    walk = [p for _, p in sorted(zip(idx, pts))]
    assert walk[0] == (0, 0, 0)
    for a, b in zip(walk, walk[1:]):
        assert sum(abs(u - v) for u, v in zip(a, b)) == 1
    end = walk[-1]  # the curve ends on a corner next to the start corner
    assert sorted(end) == [0, 0, side - 1]


@pytest.mark.parametrize("bits,level", [(3, 1), (3, 2), (4, 2), (4, 3)])
def test_hilbert_aligned_subcubes_are_contiguous_runs(bits, level):
    side, sub = 1 << bits, 1 << level
    for x0 in range(0, side, sub):
        for y0 in range(0, side, sub):
            for z0 in range(0, side, sub):
                idx = sorted(hilbert_index(x, y, z, bits) for x in range(x0, x0 + sub)
                             for y in range(y0, y0 + sub) for z in range(z0, z0 + sub))
                assert idx[-1] - idx[0] == sub ** 3 - 1 and idx[0] % sub ** 3 == 0


def test_hilbert_hand_worked_example():
    lines = [l for l in open(os.path.join(GOLDEN, "perm_worked.txt")) if not l.startswith("#")]
    kv = {l.split(":")[0]: [int(x) for x in l.split(":")[1].split()] for l in lines if ":" in l}
    g = Geom(*kv["hilbert_geometry"], order="hilbert")
    assert oracle.slot_of_token(g).tolist() == kv["hilbert_slot_of_token"]


HGEOMS = [Geom(5, 9, 7, 2, 4, 4, "hilbert"), Geom(4, 8, 8, 4, 4, 4, "hilbert"),
          Geom(3, 10, 6, 1, 8, 8, "hilbert"), Geom(1, 1, 3, 1, 1, 2, "hilbert")]


@pytest.mark.parametrize("g", HGEOMS, ids=str)
def test_hilbert_slots_fill_a_prefix_and_blocks_are_runs(g):
    s = oracle.slot_of_token(g)
    assert sorted(s.tolist()) == list(range(g.N))      # slots [0, N): only the tail pads
    L = oracle.block_len(g)
    assert L[:-1].tolist() == [g.bs] * (g.nb - 1) and L[-1] == g.N - (g.nb - 1) * g.bs
    # consecutive slots are consecutive along the curve over the enclosing cube
    bits = oracle.oracle.hilbert_bits(g)
    t, h, w = np.unravel_index(np.arange(g.N), (g.T, g.Hh, g.W))
    hidx = np.array([hilbert_index(a, b, c, bits) for a, b, c in zip(t, h, w)])
    assert np.all(np.diff(hidx[np.argsort(s)]) > 0)
    X = np.random.default_rng(20).standard_normal((1, 2, g.N, 3))
    assert np.array_equal(oracle.unreorder(oracle.reorder(X, g), g), X)


def test_hilbert_pooling_and_dense_attention():
    g = Geom(5, 9, 7, 2, 4, 4, "hilbert")
    rng = np.random.default_rng(21)
    C = rng.standard_normal((1, 1, g.nb, 4))
    X = C[:, :, oracle.slot_of_token(g) // g.bs]
    np.testing.assert_allclose(oracle.pool(oracle.reorder(X, g), g), C, atol=1e-12)
    q, k, v = (rng.standard_normal((1, 2, g.N, 16)) for _ in range(3))
    qt, kt, vt = (oracle.reorder(x, g) for x in (q, k, v))
    m = oracle.build_mask(qt, kt, g, [1.0, 1.0], 1)
    Ot, _ = oracle.attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"])
    valid = oracle.slot_valid(g)
    ref = _dense_sdpa(qt, kt, vt, g)
    np.testing.assert_allclose(Ot[:, :, valid], ref[:, :, valid], atol=1e-12)
    _mask_invariants(oracle.build_mask(qt, kt, g, [0.7, 0.9], 2), [0.7, 0.9], 2, g.nb)


# ---------------------------------------------------------------------------
# Stripe masks (Parameterized Stripe Attention for Efficient Video
# Generation, Approach: M(Tw, To, Ts, Sw, So, Ss)); the reading is stated in
# the oracle's header of that section.
# ---------------------------------------------------------------------------

# nT = 4 temporal cubes, one spatial cube
G_T4 = oracle.Geom(8, 8, 8, 2, 8, 8)
# one temporal cube, 2 x 3 spatial cubes (flattened spatial index th*3 + tw)
G_S6 = oracle.Geom(2, 16, 24, 2, 8, 8)


def test_stripe_temporal_period_hand_worked():
    """Every second frame block (w=1, o=0, s=2): catches a dropped modulo or a
    period applied to the wrong axis."""
    want = np.array([[1, 0, 1, 0], [0, 1, 0, 1], [1, 0, 1, 0], [0, 1, 0, 1]], dtype=bool)
    assert np.array_equal(oracle.stripe_keep(G_T4, (1, 0, 2, 1, 0, 0)), want)


def test_stripe_spatial_offset_sign_hand_worked():
    """ds in {-1, 0} (w=2, o=-1): the key block itself and the one just before
    it in the flattened spatial order. Catches dt/ds taken as query - key."""
    want = np.array([[1, 0, 0, 0, 0, 0],
                     [1, 1, 0, 0, 0, 0],
                     [0, 1, 1, 0, 0, 0],
                     [0, 0, 1, 1, 0, 0],
                     [0, 0, 0, 1, 1, 0],
                     [0, 0, 0, 0, 1, 1]], dtype=bool)
    assert np.array_equal(oracle.stripe_keep(G_S6, (1, 0, 0, 2, -1, 0)), want)


def test_stripe_spatial_period_hand_worked():
    """ds = 0 mod 3 (s = nW): the same cube column one cube row up or down."""
    want = np.array([[1, 0, 0, 1, 0, 0],
                     [0, 1, 0, 0, 1, 0],
                     [0, 0, 1, 0, 0, 1],
                     [1, 0, 0, 1, 0, 0],
                     [0, 1, 0, 0, 1, 0],
                     [0, 0, 1, 0, 0, 1]], dtype=bool)
    assert np.array_equal(oracle.stripe_keep(G_S6, (1, 0, 0, 1, 0, 3)), want)


SGEOMS = [oracle.Geom(8, 16, 24, 2, 8, 8), oracle.Geom(5, 9, 7, 2, 4, 8),
          oracle.Geom(21, 30, 52, 2, 8, 8), oracle.Geom(3, 17, 9, 1, 8, 8)]


@pytest.mark.parametrize("g", SGEOMS, ids=str)
def test_stripe_closed_forms(g):
    nT, nS = g.nT, g.nH * g.nW
    full = (2 * nT - 1, -(nT - 1), 0, 2 * nS - 1, -(nS - 1), 0)
    assert oracle.stripe_keep(g, full).all()
    assert np.array_equal(oracle.stripe_keep(g, (1, 0, 0, 1, 0, 0)), np.eye(g.nb, dtype=bool))
    assert not oracle.stripe_keep(g, (0, 0, 0, 1, 0, 0)).any()      # zero width
    assert not oracle.stripe_keep(g, (1, nT, 0, 1, 0, 0)).any()     # offset past the grid
    # a period no longer than the width covers every offset
    assert oracle.stripe_keep(g, (3, 5, 3, 4, -7, 2)).all()
    # temporal band alone: |tt_i - tt_j| <= 1, spatial index equal
    tt, sp = oracle.block_coords(g)
    want = (np.abs(tt[:, None] - tt[None, :]) <= 1) & (sp[:, None] == sp[None, :])
    assert np.array_equal(oracle.stripe_keep(g, (3, -1, 0, 1, 0, 0)), want)


@pytest.mark.parametrize("g", SGEOMS[:2] + SGEOMS[3:], ids=str)
def test_stripe_vectorised_equals_loops(g):
    rng = np.random.default_rng(11)
    for _ in range(12):
        prm = (int(rng.integers(0, 4)), int(rng.integers(-3, 3)), int(rng.integers(0, 4)),
               int(rng.integers(0, 7)), int(rng.integers(-6, 6)), int(rng.integers(0, 8)))
        assert np.array_equal(oracle.stripe_keep(g, prm), oracle.stripe_keep_loops(g, prm)), prm


@pytest.mark.parametrize("g", SGEOMS, ids=str)
def test_stripe_invariants(g):
    tt, sp = oracle.block_coords(g)
    # a symmetric band is a symmetric relation
    band = oracle.stripe_keep(g, (3, -1, 0, 5, -2, 0))
    assert np.array_equal(band, band.T)
    # keep depends on (dt, ds) only: equal offsets, equal decisions
    k = oracle.stripe_keep(g, (2, -1, 3, 3, -1, g.nW))
    dt = tt[None, :] - tt[:, None]
    ds = sp[None, :] - sp[:, None]
    for a in np.unique(dt):
        for c in np.unique(ds):
            sel = (dt == a) & (ds == c)
            assert k[sel].all() or not k[sel].any()
    # block coordinates cover the cube grid in cube order
    assert np.array_equal(tt * (g.nH * g.nW) + sp, np.arange(g.nb))


def test_stripe_csr_layout_matches_build_mask():
    """The stripe CSR uses build_mask's layout: with every block kept both give
    the same row_ptr, col_idx and bitmask."""
    g = oracle.Geom(5, 9, 7, 2, 4, 8)
    B, H, d = 1, 2, 8
    rng = np.random.default_rng(3)
    Qt = oracle.reorder(rng.standard_normal((B, H, g.N, d)), g)
    Kt = oracle.reorder(rng.standard_normal((B, H, g.N, d)), g)
    dense = oracle.build_mask(Qt, Kt, g, [1.0, 1.0], 0)
    nT, nS = g.nT, g.nH * g.nW
    full = (2 * nT - 1, -(nT - 1), 0, 2 * nS - 1, -(nS - 1), 0)
    st = oracle.stripe_mask(g, [full, full], B)
    for key in ("row_cnt", "row_ptr", "col_idx", "bitmask"):
        assert np.array_equal(np.asarray(st[key]), np.asarray(dense[key])), key


def test_stripe_mask_rows_heads_and_csr():
    g = oracle.Geom(8, 16, 24, 2, 8, 8)
    params = [(3, -1, 0, 5, -2, 3), (1, 0, 0, 1, 0, 0), (1, 4, 0, 1, 0, 0)]
    B, H = 2, 3
    m = oracle.stripe_mask(g, params, B)
    R = B * H * g.nb
    assert m["row_ptr"].shape == (R + 1,) and m["row_ptr"][-1] == m["col_idx"].size
    assert np.array_equal(np.diff(m["row_ptr"]), m["row_cnt"])
    bits = np.unpackbits(m["bitmask"].view(np.uint8), axis=1, bitorder="little")[:, :g.nb]
    for b in range(B):
        for h in range(H):
            rows = slice((b * H + h) * g.nb, (b * H + h + 1) * g.nb)
            assert np.array_equal(bits[rows].astype(bool), oracle.stripe_keep(g, params[h]))
    for r in range(R):
        c = m["col_idx"][m["row_ptr"][r]:m["row_ptr"][r + 1]]
        assert np.all(np.diff(c) > 0) and np.array_equal(c, np.nonzero(bits[r])[0])
    assert (m["row_cnt"][2 * g.nb:3 * g.nb] == 0).all()  # head 2: offset past the grid
    with pytest.raises(ValueError):
        oracle.stripe_mask(oracle.Geom(4, 8, 8, 4, 4, 4, order="hilbert"), params[:1], 1)


# ---------------------------------------------------------------------------
# Low-bit P.V (VC-Attention abstract: V-Smooth, ExpCast-FP8); the readings
# are stated in the oracle's header of that section.
# ---------------------------------------------------------------------------
from oracle import oracle as _o  # noqa: E402


def test_e4m3_decode_matches_torch_for_every_code():
    torch = pytest.importorskip("torch")
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = _o.e4m3_decode(np.arange(256))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    assert got[126] == 448.0 and got[1] == 2.0 ** -9 and got[8] == 2.0 ** -6 and got[56] == 1.0


def test_e4m3_encode_matches_torch_in_range_and_saturates():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
                        _o.e4m3_decode(np.arange(127)), -_o.e4m3_decode(np.arange(1, 127))])
    x = x[np.abs(x) <= 448.0].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = _o.e4m3_encode(x)
    assert np.array_equal(got, ref)  # negatives that round to zero give -0 (0x80) in both
    assert _o.e4m3_encode([500.0, 1e9, -449.0, -1e-9, -0.0])[:].tolist() == [126, 126, 254, 128, 128]
    # ties go to the even code: 1.0625 lies between 1.0 (56) and 1.125 (57)
    assert _o.e4m3_encode([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10]).tolist() == [56, 58, 0, 2]


def test_expcast_code_closed_forms():
    k = np.arange(-12, 3)
    assert np.array_equal(_o.e4m3_decode(_o.expcast_code(k)), np.exp2(k + 6.0))
    assert _o.expcast_code([0.0, 2.75, -np.inf, np.nan, -50.0, 3.0, 100.0]).tolist() == \
        [104, 126, 0, 0, 0, 126, 126]
    assert 8 * _o.EXPCAST_TAU + _o.EXPCAST_BIAS == 126  # no code clips below the threshold
    x = np.linspace(-12, 2.75, 20001)
    c = _o.expcast_code(x)
    assert np.all(np.diff(c) >= 0)                      # monotone
    rel = _o.e4m3_decode(c) / np.exp2(x + 6.0) - 1.0
    # piecewise-linear 2^x (at most +8.61 % at fraction 1/ln2 - 1) and rounding
    # to eighths (a factor 2^(+-1/16)) bound the relative error
    assert rel.max() <= (1 + 0.0861) * 2 ** (1 / 16) - 1 + 1e-9
    assert rel.min() >= 2 ** (-1 / 16) - 1 - 1e-9


def _vsmooth_case(seed=0, g=oracle.Geom(5, 9, 7, 2, 4, 8)):
    rng = np.random.default_rng(seed)
    B, H, d = 1, 2, 16
    Vt = oracle.reorder(rng.standard_normal((B, H, g.N, d)) * 3.0 + rng.standard_normal(d), g)
    return g, Vt


def test_v_smooth_error_bound_scale_and_means():
    g, Vt = _vsmooth_case()
    codes, mu, e = _o.v_smooth(Vt, g)
    valid = oracle.slot_valid(g)
    # mu_j is the plain average over the block's real tokens (slot loop)
    for j in range(g.nb):
        sl = [s for s in range(j * g.bs, (j + 1) * g.bs) if valid[s]]
        assert np.allclose(mu[0, 1, j], Vt[0, 1, sl].mean(axis=0), rtol=1e-6, atol=1e-6)
    R = np.where(valid[None, None, :, None], Vt - np.repeat(mu, g.bs, axis=2), 0.0)
    sig = np.exp2(e.astype(float))[:, :, None, None]
    amax = np.abs(R).max(axis=(2, 3))
    assert np.all(amax <= 448.0 * np.exp2(e)) and np.all(amax > 224.0 * np.exp2(e))
    deq = _o.e4m3_decode(codes) * sig
    assert np.all(np.abs(deq - R) <= np.maximum(2.0 ** -4 * np.abs(R), 2.0 ** -10 * sig) + 1e-6)
    assert np.all(codes[0, :, ~valid] == 0)
    assert np.allclose(_o.v_smooth_dequant(codes, mu, e, g), np.where(valid[None, None, :, None],
                       deq + np.repeat(mu, g.bs, axis=2), 0.0))


def test_v_smooth_is_exact_on_block_constant_values():
    g = oracle.Geom(5, 9, 7, 2, 4, 8)
    rng = np.random.default_rng(2)
    per_block = rng.standard_normal((1, 1, g.nb, 8)).astype(np.float32)
    Vt = np.repeat(per_block, g.bs, axis=2) * oracle.slot_valid(g)[None, None, :, None]
    codes, mu, e = _o.v_smooth(Vt, g)
    assert not codes.any() and e[0, 0] == 0
    assert np.array_equal(mu, per_block)


def _fp8_attention_case(seed=1, scale_v=1.0, shift_v=0.0):
    g = oracle.Geom(5, 9, 7, 2, 4, 8)
    rng = np.random.default_rng(seed)
    B, H, d = 1, 2, 16
    Qt = oracle.reorder(rng.standard_normal((B, H, g.N, d)) * 2.0, g)
    Kt = oracle.reorder(rng.standard_normal((B, H, g.N, d)), g)
    Vt = oracle.reorder(rng.standard_normal((B, H, g.N, d)) * scale_v + shift_v, g)
    R = B * H * g.nb
    sel = [np.sort(rng.choice(g.nb, size=int(rng.integers(1, g.nb + 1)), replace=False))
           for _ in range(R)]
    row_ptr = np.concatenate([[0], np.cumsum([s.size for s in sel])])
    col_idx = np.concatenate(sel)
    return g, Qt, Kt, Vt, row_ptr, col_idx


def test_fp8_attention_is_close_to_exact_attention():
    g, Qt, Kt, Vt, rp, ci = _fp8_attention_case()
    codes, mu, e = _o.v_smooth(Vt, g)
    O8, l8 = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci)
    O, l = oracle.attention(Qt, Kt, Vt, g, rp, ci)
    v = oracle.slot_valid(g)
    rel = np.linalg.norm(O8[:, :, v] - O[:, :, v]) / np.linalg.norm(O[:, :, v])
    assert rel < 0.05, rel
    # the probability codes err by at most ~+12 %/-4.3 % where they matter, so
    # the log of the denominator moves by little
    assert np.abs(l8[:, :, v] - l[:, :, v]).max() < math.log(1.12)


def test_fp8_attention_rows_are_convex_combinations_of_the_dequantised_values():
    g, Qt, Kt, Vt, rp, ci = _fp8_attention_case(seed=4)
    codes, mu, e = _o.v_smooth(Vt, g)
    O8, _ = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci)
    Vd = _o.v_smooth_dequant(codes, mu, e, g)
    v = oracle.slot_valid(g)
    B, H = Qt.shape[:2]
    for b in range(B):
        for h in range(H):
            for i in range(g.nb):
                r = (b * H + h) * g.nb + i
                keys = np.concatenate([np.arange(j * g.bs, (j + 1) * g.bs) for j in ci[rp[r]:rp[r + 1]]])
                keys = keys[v[keys]]
                o = O8[b, h, i * g.bs:(i + 1) * g.bs][v[i * g.bs:(i + 1) * g.bs]]
                assert np.all(o <= Vd[b, h, keys].max(axis=0) + 1e-9)
                assert np.all(o >= Vd[b, h, keys].min(axis=0) - 1e-9)


def test_fp8_attention_power_of_two_and_shift_equivariance():
    """Scaling V by 2 only moves the per-head exponent (same codes, O doubles
    exactly); adding one vector to every value moves only the block means (O
    moves by that vector): catches a dropped scale or a dropped mean term."""
    g, Qt, Kt, Vt, rp, ci = _fp8_attention_case(seed=3)
    v = oracle.slot_valid(g)
    c1, m1, e1 = _o.v_smooth(Vt, g)
    O1, _ = _o.attention_fp8(Qt, Kt, c1, m1, e1, g, rp, ci)
    c2, m2, e2 = _o.v_smooth(Vt * 2.0, g)
    assert np.array_equal(c1, c2) and np.array_equal(e2, e1 + 1)
    O2, _ = _o.attention_fp8(Qt, Kt, c2, m2, e2, g, rp, ci)
    assert np.array_equal(O2, 2.0 * O1)
    shift = np.array([0.5, -1.25] + [0.0] * 14)
    Vs = np.where(v[None, None, :, None], Vt + shift, 0.0)
    c3, m3, e3 = _o.v_smooth(Vs, g)
    O3, _ = _o.attention_fp8(Qt, Kt, c3, m3, e3, g, rp, ci)
    assert np.allclose(O3[:, :, v], O1[:, :, v] + shift, atol=1e-5)


def test_fp8_reference_max_is_replaced_when_a_later_block_dominates():
    """A row whose second block scores 20 (log2 units) above its first: the
    first block's weight falls to 0 and the output is the second block's own
    low-bit average. Without replacing the reference the codes would clip at
    448 and the output would move."""
    g = oracle.Geom(4, 8, 8, 4, 4, 4)  # nb = 4 full blocks of 64
    rng = np.random.default_rng(7)
    d = 8
    Qt = np.zeros((1, 1, g.Npad, d)); Qt[..., 0] = 1.0
    Kt = rng.standard_normal((1, 1, g.Npad, d)) * 0.1
    boost = 20.0 * math.sqrt(d) / math.log2(math.e)
    Kt[0, 0, 2 * g.bs:3 * g.bs, 0] += boost
    Vt = rng.standard_normal((1, 1, g.Npad, d))
    codes, mu, e = _o.v_smooth(Vt, g)
    R = g.nb
    rp = np.arange(R + 1) * 2
    ci = np.tile([0, 2], R)
    O8, _ = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci, blocks=[(0, 0, 0)])
    only2, _ = _o.attention_fp8(Qt, Kt, codes, mu, e, g, np.arange(R + 1), np.full(R, 2),
                                blocks=[(0, 0, 0)])
    sl = slice(0, g.bs)
    assert np.allclose(O8[0, 0, sl], only2[0, 0, sl], atol=1e-4)


# Reference rule of ExpCast-FP8 (VC-Attention abstract: codes from one
# multiply-add inside the online softmax). Hand-worked rows: block maxima in
# log2 units, in col_idx order, and the reference in force at each block.
_REFERENCE_ROWS = [
    ([0.0, 2.70, 2.80], [0.0, 0.0, 2.80]),    # 2.70 keeps; 2.80 is more than 2.75 above 0
    ([0.0, 2.75], [0.0, 0.0]),                # exactly 2.75 above keeps (strict >)
    ([0.0, 2.70, 5.50], [0.0, 0.0, 5.50]),
    ([1.0, -3.0, 3.76, 3.70], [1.0, 1.0, 3.76, 3.76]),
    ([1.0, 3.74, 6.5, 9.2501], [1.0, 1.0, 6.5, 9.2501]),
    ([-4.0, -9.0, -1.25, -1.2499], [-4.0, -4.0, -4.0, -1.2499]),
]


def _reference_pins_hold(rule) -> bool:
    for bm, want in _REFERENCE_ROWS:
        got = rule(np.array(bm)[:, None])[:, 0]
        if not np.array_equal(got, np.array(want)):
            return False
    return True


def test_expcast_reference_hand_worked_rows():
    assert _reference_pins_hold(_o.expcast_reference)
    # invert takes the other decision at the marked block only
    inv = np.zeros((3, 1), dtype=bool)
    inv[1, 0] = True
    assert _o.expcast_reference(np.array([[0.0], [2.70], [2.80]]), inv)[:, 0].tolist() == \
        [0.0, 2.70, 2.70]


def test_expcast_reference_pins_catch_plausible_slips():
    """The pins fail for a >= comparison and for a rule that compares with
    the running maximum instead of the reference."""
    def ge_rule(bm):
        ref = np.empty_like(bm)
        ref[0] = bm[0]
        for k in range(1, len(bm)):
            ref[k] = np.where(bm[k] >= ref[k - 1] + 2.75, bm[k], ref[k - 1])
        return ref

    def running_max_rule(bm):
        ref = np.empty_like(bm)
        ref[0] = bm[0]
        run = bm[0].copy()
        for k in range(1, len(bm)):
            ref[k] = np.where(bm[k] > run + 2.75, bm[k], ref[k - 1])
            run = np.maximum(run, bm[k])
        return ref

    assert not _reference_pins_hold(ge_rule)
    assert not _reference_pins_hold(running_max_rule)


def _one_row_case(xs, vals, d=8):
    """One mask row over blocks 0..len(xs)-1 of a 4-block layer of 64-token
    cubes: every key of block j scores xs[j] (log2 units) against every query,
    and every value of block j is vals[j] (so V-Smooth stores zero codes and
    the block means carry the values)."""
    g = Geom(4, 8, 8, 4, 4, 4)
    c2 = math.log2(math.e) / math.sqrt(d)
    Qt = np.zeros((1, 1, g.Npad, d))
    Qt[..., 0] = 1.0
    Kt = np.zeros((1, 1, g.Npad, d))
    Vt = np.zeros((1, 1, g.Npad, d))
    for j, (x, v) in enumerate(zip(xs, vals)):
        Kt[0, 0, j * g.bs:(j + 1) * g.bs, 0] = x / c2
        Vt[0, 0, j * g.bs:(j + 1) * g.bs] = v
    codes, mu, e = _o.v_smooth(Vt, g)
    assert not codes.any()
    n = len(xs)
    rp = np.array([0] + [n] * g.nb)
    ci = np.arange(n)
    return g, Qt, Kt, codes, mu, e, rp, ci


@pytest.mark.parametrize("xs,refs", [([0.0, 2.70, 2.80], [2.80, 2.80, 2.80]),
                                     ([0.0, 2.70, 5.50], [5.50, 5.50, 5.50]),
                                     ([0.0, -2.0, 2.70], [0.0, 0.0, 0.0])])
def test_fp8_attention_hand_worked_reference_rows(xs, refs):
    """O and lse of one row worked by hand from the code table: a block at x
    (log2 units) against the reference it is coded under (its own m at the
    time) takes code rint(8(x - m) + 104), and the accumulators carry a factor
    2^(m - m_final) for every later replacement."""
    vals = [np.full(8, 1.0), np.full(8, -2.0), np.full(8, 5.0)]
    g, Qt, Kt, codes, mu, e, rp, ci = _one_row_case(xs, vals)
    m_at = _o.expcast_reference(np.array(xs)[:, None])[:, 0]
    # codes by hand: 104 at the reference, 8 * 2.70 + 104 = 125.6 -> 126 (448),
    # 8 * -2 + 104 = 88 (16)
    table = {104: 64.0, 126: 448.0, 88: 16.0}
    w = []
    for x, m in zip(xs, m_at):
        c = int(round(8 * (x - m) + 104))
        w.append(64 * table[c] * 2.0 ** (m - refs[-1]))
    L = sum(w)
    want_o = sum(wi * v for wi, v in zip(w, vals)) / L
    want_lse = math.log(L) + (refs[-1] - 6.0) * math.log(2.0)
    O8, l8 = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci, blocks=[(0, 0, 0)])
    assert np.allclose(O8[0, 0, :g.bs], want_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(l8[0, 0, :g.bs], want_lse, rtol=1e-12, atol=1e-12)
    assert list(m_at) == [0.0, 0.0, refs[-1]] or xs[-1] < 2.75


def test_fp8_flip_bound_covers_a_code_on_its_rounding_boundary():
    """Block 1 scores sit on the boundary between codes 95 and 96
    (8 * -1.0625 + 104 = 95.5): nudging them either way flips all 64 codes.
    The margin report flags them, its bound covers the actual move of O and
    lse, and is within a small factor of it."""
    vals = [np.full(8, 1.0), np.full(8, -2.0)]
    outs = []
    for eps in (1e-9, -1e-9):
        g, Qt, Kt, codes, mu, e, rp, ci = _one_row_case([0.0, -1.0625 + eps], vals)
        O8, l8, dg = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci, blocks=[(0, 0, 0)], diag=True)
        outs.append((O8[0, 0, 0], l8[0, 0, 0], dg["flip_o"][0, 0, 0], dg["flip_lse"][0, 0, 0],
                     dg["thr_near"][0, 0, 0]))
    (o1, l1, f1, fl1, t1), (o2, l2, f2, fl2, t2) = outs
    move = np.abs(o1 - o2)
    assert move.min() > 1e-3                       # the flip is real
    assert np.all(move <= f1) and np.all(move <= f2)
    assert np.all(f1 <= 3.0 * move) and np.all(f2 <= 3.0 * move)
    # (the lse bound is exact for a flip that lowers the sum: equal up to rounding)
    assert abs(l1 - l2) <= min(fl1, fl2) + 1e-12 and max(fl1, fl2) <= 3.0 * abs(l1 - l2)
    assert t1 == 0 and t2 == 0
    # away from any boundary the report is empty
    g, Qt, Kt, codes, mu, e, rp, ci = _one_row_case([0.0, -1.0], vals)
    _, _, dg = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci, blocks=[(0, 0, 0)], diag=True)
    assert not dg["flip_o"].any() and not dg["flip_lse"].any()


def test_fp8_threshold_report_and_the_other_decision():
    """A block maximum exactly 2.75 above the reference is flagged; the
    inverted decision reproduces a run that replaced the reference there."""
    vals = [np.full(8, 1.0), np.full(8, -2.0)]
    g, Qt, Kt, codes, mu, e, rp, ci = _one_row_case([0.0, 2.75], vals)
    O8, l8, dg = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci, blocks=[(0, 0, 0)], diag=True)
    assert np.all(dg["thr_near"][0, 0, :g.bs] == 1) and np.all(dg["thr_first"][0, 0, :g.bs] == 1)
    inv = np.zeros((2, g.bs), dtype=bool)
    inv[1] = True
    Oi, li = _o.attention_fp8(Qt, Kt, codes, mu, e, g, rp, ci, blocks=[(0, 0, 0)],
                              invert={(0, 0, 0): inv})
    # by hand: kept -> codes 104 and 126 (64, 448); replaced -> block 0 keeps
    # the code it took under the old reference (104: 64), rescaled by
    # 2^(0 - 2.75), and block 1 takes 104 (64)
    w0 = 64.0 * 2.0 ** -2.75
    kept = (64 * 1.0 + 448 * -2.0) / (64 + 448)
    repl = (w0 * 1.0 + 64 * -2.0) / (w0 + 64)
    assert np.allclose(O8[0, 0, 0], kept, atol=1e-12)
    assert np.allclose(Oi[0, 0, 0], repl, atol=1e-12)
    assert np.isclose(li[0, 0, 0], math.log(64 * (w0 + 64)) + (2.75 - 6.0) * math.log(2.0))
