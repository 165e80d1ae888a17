"""Plain fp64 CPU oracle for training-free Top-p block-sparse video attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code with the CUDA library and never imports it.

What it computes, step by step, and the passages each step follows:

* FVAttn abstract ("video-aware block organization"): tokens of a T x Hh x W
  latent grid are grouped into spatio-temporal cubes of ct x ch x cw tokens;
  each cube is one block of ``bs = ct*ch*cw`` slots. ``reorder``/``unreorder``.
* FVAttn abstract ("Top-p routing, a Top-k safety floor"): each query block
  scores every key block with the softmax of mean-pooled Q and K blocks,
  ``softmax_j(Qbar_i . Kbar_j / sqrt(d))``, and keeps the smallest prefix of key
  blocks, in descending score order, whose cumulative mass reaches p, but never
  fewer than k blocks. ``pool``, ``block_probs``, ``select_row``, ``build_mask``.
* FVAttn abstract (the sparse attention that the mask drives): for every query
  of block i, exact softmax attention over the keys of the selected blocks
  only. ``attention``.

Readings where the pages are silent (each listed in the design notes):

* ragged grids are padded up to whole cubes; inside an edge cube the real
  tokens come first, row-major (t, h, w) over the cube's real sub-box, and the
  padding slots (zeros) fill the tail of the block, so every block's real
  slots are a prefix of it;
* cubes are ordered row-major over the cube grid (t, h, w) and tokens row-major
  inside a cube (for a complete cube: offset ((t%ct)*ch + h%ch)*cw + w%cw);
* pooled means divide by the number of valid tokens of the block;
* no length correction of partial blocks, no forced diagonal, no causality;
* Top-p takes the shortest prefix with cumulative mass >= p (inclusive);
  when the floating-point sum never reaches p, or p >= 1, every block is kept;
* ties between equal scores go to the lower key-block index;
* k larger than the number of key blocks keeps every block;
* padding query slots produce O = 0 and lse = 0.

Parity is pinned by tests/test_oracle.py (brute force, closed forms,
library routines, invariants); no function here is "parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Geom:
    """Grid and block geometry (FVAttn abstract: video-aware block organization).

    order "cube": blocks are ct x ch x cw cubes (an edge cube keeps its real
    tokens in its first slots and padding in the rest).
    order "hilbert": tokens follow a 3-D Hilbert curve over (t, h, w) and every
    run of bs = ct*ch*cw consecutive tokens is a block; only the last block
    can be partial (DFSAttn: Hilbert-curve token reordering)."""

    T: int
    Hh: int
    W: int
    ct: int
    ch: int
    cw: int
    order: str = "cube"

    @property
    def N(self):
        return self.T * self.Hh * self.W

    @property
    def bs(self):
        return self.ct * self.ch * self.cw

    @property
    def nT(self):
        return -(-self.T // self.ct)

    @property
    def nH(self):
        return -(-self.Hh // self.ch)

    @property
    def nW(self):
        return -(-self.W // self.cw)

    @property
    def nb(self):
        if self.order == "hilbert":
            return -(-self.N // self.bs)
        return self.nT * self.nH * self.nW

    @property
    def Npad(self):
        return self.nb * self.bs


# ---------------------------------------------------------------------------
# Video-aware block organization (FVAttn abstract)
# ---------------------------------------------------------------------------

def hilbert_index(x, y, z, bits: int) -> int:
    """Position of point (x, y, z) of a 2^bits cube along a 3-D Hilbert curve.

    J. Skilling, "Programming the Hilbert curve" (AIP Conf. Proc. 707, 2004):
    turn the coordinates into the curve's "transposed" form by undoing the
    reflections and axis swaps level by level from the top bit down, Gray-encode
    across axes, then read the index off the transposed bits, top level first,
    one bit per axis in axis order."""
    X = [int(x), int(y), int(z)]
    n = 3
    M = 1 << (bits - 1)
    Q = M
    while Q > 1:
        P = Q - 1
        for i in range(n):
            if X[i] & Q:
                X[0] ^= P                      # reflect the low bits of axis 0
            else:
                t = (X[0] ^ X[i]) & P          # swap the low bits of axes 0 and i
                X[0] ^= t
                X[i] ^= t
        Q >>= 1
    for i in range(1, n):                      # Gray encode across axes
        X[i] ^= X[i - 1]
    t = 0
    Q = M
    while Q > 1:
        if X[n - 1] & Q:
            t ^= Q - 1
        Q >>= 1
    for i in range(n):
        X[i] ^= t
    h = 0
    for b in range(bits - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((X[i] >> b) & 1)
    return h


def hilbert_bits(g: Geom) -> int:
    """Bits per axis of the smallest power-of-two cube holding the grid."""
    side = max(g.T, g.Hh, g.W)
    return max(1, (side - 1).bit_length())


def slot_of_token(g: Geom) -> np.ndarray:
    """Slot of every raster token ``n = (t*Hh + h)*W + w``.

    Hilbert order: slot = rank of the token's Hilbert index among all tokens.
    Cube order: the token lands in cube ``blk = (t//ct * nH + h//ch) * nW + w//cw``.
    The cube's real sub-box has extents ``vt = min(ct, T - t//ct*ct)`` (and vh,
    vw alike); the token's in-cube offset is ``((t%ct)*vh + h%ch)*vw + w%cw``,
    its rank row-major over that sub-box, so the real tokens of a block fill
    slots ``[0, vt*vh*vw)`` and padding the rest; slot = blk*bs + offset.
    For a complete cube this is ``((t%ct)*ch + h%ch)*cw + w%cw``.
    """
    if g.order == "hilbert":
        # the token's rank along the curve among the grid's tokens
        bits = hilbert_bits(g)
        idx = np.array([hilbert_index(t, h, w, bits) for t in range(g.T) for h in range(g.Hh)
                        for w in range(g.W)], dtype=np.int64)
        slot = np.empty(g.N, dtype=np.int64)
        slot[np.argsort(idx, kind="stable")] = np.arange(g.N)
        return slot
    t, h, w = np.meshgrid(np.arange(g.T), np.arange(g.Hh), np.arange(g.W), indexing="ij")
    t, h, w = t.ravel(), h.ravel(), w.ravel()
    th, tw = h // g.ch, w // g.cw
    blk = ((t // g.ct) * g.nH + th) * g.nW + tw
    vh = np.minimum(g.ch, g.Hh - th * g.ch)   # real extents of the token's cube
    vw = np.minimum(g.cw, g.W - tw * g.cw)
    off = ((t % g.ct) * vh + (h % g.ch)) * vw + (w % g.cw)
    return (blk * g.bs + off).astype(np.int64)


def slot_of_token_loops(g: Geom) -> np.ndarray:
    """The same permutation written as explicit loops over cubes and in-cube
    positions (small grids only): inside every cube, hand out its first slots
    to the real tokens in row-major (t, h, w) order; the rest is padding."""
    out = np.full(g.N, -1, dtype=np.int64)
    blk = 0
    for tt in range(g.nT):
        for th in range(g.nH):
            for tw in range(g.nW):
                s = blk * g.bs
                for lt in range(g.ct):
                    for lh in range(g.ch):
                        for lw in range(g.cw):
                            t, h, w = tt * g.ct + lt, th * g.ch + lh, tw * g.cw + lw
                            if t < g.T and h < g.Hh and w < g.W:
                                out[(t * g.Hh + h) * g.W + w] = s
                                s += 1
                blk += 1
    return out


def slot_valid(g: Geom) -> np.ndarray:
    """Boolean [Npad]: True where the slot holds a real token."""
    v = np.zeros(g.Npad, dtype=bool)
    v[slot_of_token(g)] = True
    return v


def block_len(g: Geom) -> np.ndarray:
    """Number of real tokens in every block, by counting valid slots."""
    return slot_valid(g).reshape(g.nb, g.bs).sum(axis=1).astype(np.int64)


def reorder(X: np.ndarray, g: Geom) -> np.ndarray:
    """[B,H,N,d] raster -> [B,H,Npad,d] cube order, padding slots zero (fp64)."""
    B, H, N, d = X.shape
    assert N == g.N
    Xt = np.zeros((B, H, g.Npad, d), dtype=np.float64)
    Xt[:, :, slot_of_token(g)] = X
    return Xt


def unreorder(Xt: np.ndarray, g: Geom) -> np.ndarray:
    """[B,H,Npad,d] cube order -> [B,H,N,d] raster; padding slots are dropped."""
    return np.asarray(Xt, dtype=np.float64)[:, :, slot_of_token(g)]


# ---------------------------------------------------------------------------
# Block scoring and Top-p / Top-k routing (FVAttn abstract)
# ---------------------------------------------------------------------------

def pool(Xt: np.ndarray, g: Geom) -> np.ndarray:
    """Mean of the real tokens of every block: [B,H,Npad,d] -> [B,H,nb,d]."""
    B, H, _, d = Xt.shape
    valid = slot_valid(g).reshape(g.nb, g.bs)
    blocks = np.asarray(Xt, dtype=np.float64).reshape(B, H, g.nb, g.bs, d)
    sums = (blocks * valid[None, None, :, :, None]).sum(axis=3)
    return sums / block_len(g)[None, None, :, None]


def block_probs(Qbar: np.ndarray, Kbar: np.ndarray) -> np.ndarray:
    """Row softmax over key blocks of ``Qbar Kbar^T / sqrt(d)``: [..,nb,d] -> [..,nb,nb]."""
    d = Qbar.shape[-1]
    S = np.matmul(Qbar, np.swapaxes(Kbar, -1, -2)) / math.sqrt(d)
    S = S - S.max(axis=-1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=-1, keepdims=True)


def select_row(P: np.ndarray, p: float, k: int):
    """Top-p with a Top-k floor on one row of block probabilities.

    Sort descending (ties: lower index first), take the shortest prefix whose
    cumulative mass reaches p, then at least k entries, at most all of them.
    Returns (selected indices ascending, info) where info carries the
    quantities the exemption rules need.
    """
    P = np.asarray(P, dtype=np.float64)
    nkb = P.shape[0]
    order = np.lexsort((np.arange(nkb), -P))
    c = np.cumsum(P[order])
    if p >= 1.0:
        n_p = nkb
    else:
        hit = np.nonzero(c >= p)[0]
        n_p = int(hit[0]) + 1 if hit.size else nkb
    n = min(nkb, max(int(k), n_p))
    sel = np.sort(order[:n])
    info = {
        "n_p": n_p,
        "n": n,
        "c_at": float(c[n_p - 1]),
        "c_before": float(c[n_p - 2]) if n_p >= 2 else 0.0,
        "order": order,
    }
    return sel, info


def build_mask(Qt: np.ndarray, Kt: np.ndarray, g: Geom, top_p, top_k: int,
               boundary_tol: float = 1e-4) -> dict:
    """Pool, score, select every (b, h, query block) row; emit bitmask and CSR.

    Rows are flattened as r = (b*H + h)*nb + i. ``col_idx`` is ascending inside
    each row. Bit j of a row lives in word j//32 at position j%32.
    ``boundary`` marks rows whose cumulative mass at the cut lies within
    ``boundary_tol`` of p (the only rows where another correct fp64
    evaluation may cut elsewhere).
    """
    B, H = Qt.shape[:2]
    nb = g.nb
    words = -(-nb // 32)
    Pm = block_probs(pool(Qt, g), pool(Kt, g))  # [B,H,nb,nb]
    R = B * H * nb
    row_cnt = np.zeros(R, dtype=np.int64)
    bitmask = np.zeros((R, words), dtype=np.uint32)
    boundary = np.zeros(R, dtype=bool)
    cols = []
    for b in range(B):
        for h in range(H):
            p = float(top_p[h])
            for i in range(nb):
                r = (b * H + h) * nb + i
                sel, info = select_row(Pm[b, h, i], p, top_k)
                row_cnt[r] = sel.size
                cols.append(sel)
                bits = np.zeros(words * 32, dtype=bool)
                bits[sel] = True  # bit j%32 of word j//32, least significant first
                bitmask[r] = np.packbits(bits, bitorder="little").view("<u4")
                boundary[r] = (abs(info["c_at"] - p) <= boundary_tol
                               or abs(info["c_before"] - p) <= boundary_tol)
    row_ptr = np.zeros(R + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(row_cnt)
    col_idx = np.concatenate(cols).astype(np.int64) if cols else np.zeros(0, np.int64)
    return {"probs": Pm, "row_cnt": row_cnt, "row_ptr": row_ptr, "col_idx": col_idx,
            "bitmask": bitmask, "boundary": boundary}


def lpt_order(row_cnt: np.ndarray, nb: int) -> np.ndarray:
    """Work order, longest first, head by head (FVAttn abstract: uneven
    per-head workloads; doing the heaviest work first limits the straggler
    tail). Heads (b, h) are taken by their total selected-block count,
    descending (ties: lower head index first); inside a head, its nb rows by
    selected-block count, descending (ties: lower row index first).

    Reading: longest-first at the granularity of heads, then of rows, so the
    rows worked on at the same time share one head's keys and values."""
    cnt = np.asarray(row_cnt, dtype=np.int64)
    R = cnt.size
    BH = R // nb
    tot = cnt.reshape(BH, nb).sum(axis=1)
    head_rank = np.empty(BH, dtype=np.int64)
    head_rank[np.lexsort((np.arange(BH), -tot))] = np.arange(BH)
    rows = np.arange(R)
    return np.lexsort((rows, -cnt, head_rank[rows // nb])).astype(np.int64)


# ---------------------------------------------------------------------------
# Block-sparse attention (FVAttn abstract)
# ---------------------------------------------------------------------------

def attention(Qt, Kt, Vt, g: Geom, row_ptr, col_idx, blocks=None):
    """Exact softmax attention of every real query slot over the real key slots
    of its block's selected key blocks.

    ``blocks``: optional iterable of (b, h, i) query blocks to compute; others
    are left NaN. Returns (Ot [B,H,Npad,d], lse [B,H,Npad]) in fp64 where
    ``lse = log sum_k exp(q.k / sqrt(d))`` (natural log). Padding query slots
    give O = 0 and lse = 0.
    """
    Qt = np.asarray(Qt, dtype=np.float64)
    Kt = np.asarray(Kt, dtype=np.float64)
    Vt = np.asarray(Vt, dtype=np.float64)
    B, H, Npad, d = Qt.shape
    nb, bs = g.nb, g.bs
    valid = slot_valid(g)
    Ot = np.full((B, H, Npad, d), np.nan)
    lse = np.full((B, H, Npad), np.nan)
    if blocks is None:
        blocks = [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    scale = 1.0 / math.sqrt(d)
    for (b, h, i) in blocks:
        r = (b * H + h) * nb + i
        sel = np.asarray(col_idx[row_ptr[r]:row_ptr[r + 1]], dtype=np.int64)
        key_slots = (sel[:, None] * bs + np.arange(bs)[None, :]).ravel()
        key_slots = key_slots[valid[key_slots]]
        q_slots = np.arange(i * bs, (i + 1) * bs)
        q = Qt[b, h, q_slots]
        s = (q @ Kt[b, h, key_slots].T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        o = (e / l) @ Vt[b, h, key_slots]
        qv = valid[q_slots]
        o[~qv] = 0.0
        ls = (m + np.log(l))[:, 0]
        ls[~qv] = 0.0
        Ot[b, h, q_slots] = o
        lse[b, h, q_slots] = ls
    return Ot, lse


def forward(q, k, v, g: Geom, top_p, top_k: int):
    """The whole path on raster inputs: reorder, route, attend, unreorder."""
    qt, kt, vt = reorder(q, g), reorder(k, g), reorder(v, g)
    m = build_mask(qt, kt, g, top_p, top_k)
    ot, lse = attention(qt, kt, vt, g, m["row_ptr"], m["col_idx"])
    return unreorder(ot, g), m, lse


# ---------------------------------------------------------------------------
# Stripe masks (Parameterized Stripe Attention for Efficient Video Generation,
# Approach: a six-parameter mask M(Tw, To, Ts, Sw, So, Ss) of periodic
# diagonal stripes, from spatio-temporal locality and RoPE-3D periodicity)
# ---------------------------------------------------------------------------
#
# Reading (the page names the parameters but prints no formula): T* act on the
# temporal offset between the key block and the query block, S* on their
# spatial offset; w is a stripe's width, o its offset, s its period (0: the
# stripe occurs once). On the cube grid, with a block's coordinates (tt, th,
# tw) and its flattened spatial index sp = th*nW + tw,
#   dt = tt_key - tt_query,   ds = sp_key - sp_query,
#   x lies in stripe (w, o, s)  <=>  0 <= x - o < w            (s = 0)
#                                    (x - o) mod s < w          (s > 0)
#   keep(query block, key block) <=> dt in (Tw, To, Ts) and ds in (Sw, So, Ss).
# A band of half-width r around the diagonal is (w, o, s) = (2r+1, -r, 0); a
# band that recurs every nW blocks of the flattened spatial index (the same
# column one cube row up or down) uses s = nW.

def in_stripe(x, w: int, o: int, s: int):
    """x (int or int array) lies in the stripe of width w starting at offset o,
    repeated with period s (s = 0: not repeated)."""
    x = np.asarray(x, dtype=np.int64)
    if s == 0:
        return (x - o >= 0) & (x - o < w)
    return np.mod(x - o, s) < w  # numpy's mod is non-negative for s > 0


def block_coords(g: Geom):
    """(tt, sp) of every block in cube order: its temporal cube coordinate and
    its flattened spatial cube index th*nW + tw."""
    j = np.arange(g.nb, dtype=np.int64)
    tt = j // (g.nH * g.nW)
    sp = j % (g.nH * g.nW)
    return tt, sp


def stripe_keep(g: Geom, prm) -> np.ndarray:
    """[nb, nb] bool keep matrix of one head, rows = query blocks."""
    Tw, To, Ts, Sw, So, Ss = (int(v) for v in prm)
    tt, sp = block_coords(g)
    dt = tt[None, :] - tt[:, None]
    ds = sp[None, :] - sp[:, None]
    return in_stripe(dt, Tw, To, Ts) & in_stripe(ds, Sw, So, Ss)


def stripe_keep_loops(g: Geom, prm) -> np.ndarray:
    """Same as stripe_keep with plain loops over the cube grid (small cases)."""
    Tw, To, Ts, Sw, So, Ss = (int(v) for v in prm)

    def inside(x, w, o, s):
        return (0 <= x - o < w) if s == 0 else ((x - o) % s < w)

    keep = np.zeros((g.nb, g.nb), dtype=bool)
    for qt_ in range(g.nT):
        for qh in range(g.nH):
            for qw in range(g.nW):
                i = (qt_ * g.nH + qh) * g.nW + qw
                for kt_ in range(g.nT):
                    for kh in range(g.nH):
                        for kw in range(g.nW):
                            j = (kt_ * g.nH + kh) * g.nW + kw
                            dt = kt_ - qt_
                            ds = (kh * g.nW + kw) - (qh * g.nW + qw)
                            keep[i, j] = inside(dt, Tw, To, Ts) and inside(ds, Sw, So, Ss)
    return keep


def csr_from_keep(keep_rows: np.ndarray) -> dict:
    """Bitmask and CSR of a stack of keep rows [R, nb] (same layout as
    build_mask: bit j%32 of word j//32, col_idx ascending inside a row)."""
    keep_rows = np.asarray(keep_rows, dtype=bool)
    R, nb = keep_rows.shape
    words = -(-nb // 32)
    bits = np.zeros((R, words * 32), dtype=bool)
    bits[:, :nb] = keep_rows
    bitmask = np.packbits(bits, axis=1, bitorder="little").view("<u4").reshape(R, words)
    row_cnt = keep_rows.sum(axis=1).astype(np.int64)
    row_ptr = np.zeros(R + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(row_cnt)
    col_idx = np.nonzero(keep_rows)[1].astype(np.int64)  # row-major: ascending j per row
    return {"row_cnt": row_cnt, "row_ptr": row_ptr, "col_idx": col_idx, "bitmask": bitmask}


def stripe_mask(g: Geom, params, B: int) -> dict:
    """Stripe mask of every (b, h, query block) row: params[h] = (Tw, To, Ts,
    Sw, So, Ss) for head h; rows r = (b*H + h)*nb + i as in build_mask."""
    if g.order != "cube":
        raise ValueError("stripe masks are defined on the cube grid")
    per_head = [stripe_keep(g, prm) for prm in params]
    rows = np.concatenate([per_head[h] for _ in range(B) for h in range(len(params))], axis=0)
    return csr_from_keep(rows)


# ---------------------------------------------------------------------------
# Low-bit P.V (VC-Attention: Value Smoothing and Softmax Casting for Low-bit
# Attention, abstract: V-Smooth and ExpCast-FP8)
# ---------------------------------------------------------------------------
#
# Readings (the abstract gives the ideas, not the formulas):
# * E4M3 is the "fn" encoding: sign bit 7, exponent bits 3..6 with bias 7,
#   mantissa bits 0..2, exponent 0 subnormal (M/8 * 2^-6), code 0x7F NaN, no
#   infinities, largest finite 448. Encoding rounds to nearest, ties to the
#   even code, saturates at +-448, and keeps the sign of a negative value
#   that rounds to zero (code 0x80).
# * V-Smooth: for every key block j, mu_j = mean of V over the block's real
#   tokens; the residual R = V - mu_j (zero on padding slots) is quantised to
#   E4M3 with one power-of-two scale per (batch, head), sigma = 2^e with e the
#   smallest integer such that max|R| <= 448 * 2^e (e = 0 when R is all zero),
#   so that one fp32 accumulator serves every block. The mean comes back
#   through the per-block row sums: sum_j l_j mu_j with l_j the sum of the
#   block's probabilities. mu_j, R and the scaling are evaluated in fp32 (the
#   kernels' precision), the quantisation decision on the fp32 values. The
#   page's online clustering of value tokens is not built: cube blocks already
#   hold spatio-temporal neighbours.
# * ExpCast-FP8: the probability code of a log2-domain score x taken relative
#   to the row's reference maximum (x <= 0 at the reference) is
#   c = clamp(rint(8x + 104), 0, 126): one multiply-add puts the integer part
#   of x + 13 into the exponent field and eighths of its fraction into the
#   mantissa field, so decode(c) interpolates 2^(x+6) linearly between powers
#   of two (exact where 8x is an integer and -12 <= x <= 2.75). The reference
#   maps to 2^6 rather than 1 so that normal codes cover 12 octaves below it
#   and 2.75 above it; the factor cancels in the normalisation and lse
#   removes it.
# * Reference maximum: the row maximum of the first selected block; a later
#   block whose maximum exceeds the reference by more than 2.75 (log2 units)
#   replaces it (the accumulators are rescaled by 2^(old - new)); a block
#   whose maximum lies exactly 2.75 above keeps it. The rule is forced by the
#   online form the abstract gives (the mean comes back through the row sum
#   that the online softmax keeps): codes are taken block by block, before
#   later blocks are seen, against a reference that only moves forward, and
#   2.75 is the headroom of the code range above the reference
#   ((126 - 104) / 8), the largest jump that needs no rescale without a code
#   clipping at 448. With low-bit codes the reference changes the codes (the
#   fraction of 8x moves with it), so the rule, applied to the selected blocks
#   in ascending key-block order, is part of the definition.

E4M3_MAX = 448.0


def e4m3_decode(code) -> np.ndarray:
    """Values of E4M3 codes (0..255)."""
    c = np.asarray(code, dtype=np.int64)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where(c & 0x80, -mag, mag)


_E4M3_POS = e4m3_decode(np.arange(127))  # finite non-negative values, codes 0..126, ascending


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 code of x (ties to the even code), saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, ax), 1, 126)
    lo = hi - 1
    dlo = ax - _E4M3_POS[lo]
    dhi = _E4M3_POS[hi] - ax
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(ax >= _E4M3_POS[126], 126, code)
    # a negative value keeps its sign bit even when it rounds to zero (-0)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


EXPCAST_BIAS = 104.0  # code of the reference maximum (value 2^6)
EXPCAST_TAU = 2.75    # reference replacement threshold, log2 units (8 * 2.75 + 104 = 126)


def expcast_code(x) -> np.ndarray:
    """ExpCast-FP8 probability code of log2-domain scores x relative to the
    reference maximum (reading above)."""
    y = np.rint(8.0 * np.asarray(x, dtype=np.float64) + EXPCAST_BIAS)
    return np.clip(np.nan_to_num(y, nan=0.0, neginf=0.0), 0, 126).astype(np.int64)


def v_smooth(Vt: np.ndarray, g: Geom):
    """V-Smooth quantisation of cube-ordered values Vt [B,H,Npad,d].

    Returns (codes uint8 [B,H,Npad,d], mu fp32 [B,H,nb,d], e int [B,H])."""
    B, H, Npad, d = Vt.shape
    nb, bs = g.nb, g.bs
    valid = slot_valid(g)
    V32 = np.asarray(Vt, dtype=np.float32).reshape(B, H, nb, bs, d)
    vmask = valid.reshape(nb, bs)[None, None, :, :, None]
    cnt = valid.reshape(nb, bs).sum(axis=1).astype(np.float64)[None, None, :, None]
    mu = (np.where(vmask, V32.astype(np.float64), 0.0).sum(axis=3) / cnt).astype(np.float32)
    R = np.where(vmask, V32 - mu[:, :, :, None, :], np.float32(0.0)).astype(np.float32)
    e = np.zeros((B, H), dtype=np.int64)
    codes = np.zeros((B, H, nb, bs, d), dtype=np.uint8)
    for b in range(B):
        for h in range(H):
            amax = float(np.abs(R[b, h]).max())
            if amax > 0.0:
                k = int(math.ceil(math.log2(amax / E4M3_MAX)))
                while amax > E4M3_MAX * 2.0 ** k:  # guard the log2 rounding
                    k += 1
                while k > -149 and amax <= E4M3_MAX * 2.0 ** (k - 1):
                    k -= 1
                e[b, h] = k
            scaled = (R[b, h] * np.float32(2.0 ** -int(e[b, h]))).astype(np.float32)
            codes[b, h] = e4m3_encode(scaled)
    return codes.reshape(B, H, Npad, d), mu, e


def v_smooth_dequant(codes: np.ndarray, mu: np.ndarray, e: np.ndarray, g: Geom) -> np.ndarray:
    """sigma * decode(codes) + mu_j on real slots, 0 on padding: the values the
    low-bit path effectively attends to."""
    B, H, Npad, d = codes.shape
    valid = slot_valid(g)
    R = e4m3_decode(codes) * np.exp2(e.astype(np.float64))[:, :, None, None]
    Vd = R + np.repeat(mu.astype(np.float64), g.bs, axis=2)
    return np.where(valid[None, None, :, None], Vd, 0.0)


def expcast_reference(block_max, invert=None) -> np.ndarray:
    """Reference maximum in force for each block of a row (reading above).

    block_max [n, rows]: the rows' maxima over the real keys of their n
    selected blocks, in col_idx order (log2 units). Returns [n, rows]: ref[0]
    = block_max[0]; ref[k] = block_max[k] if block_max[k] > ref[k-1] + 2.75,
    else ref[k-1]. ``invert`` (bool [n, rows]) takes the opposite decision at
    the marked (block, row) pairs (block 0 has no decision): used to follow
    a run that decided a near-threshold comparison the other way."""
    bm = np.asarray(block_max, dtype=np.float64)
    ref = np.empty_like(bm)
    if bm.shape[0] == 0:
        return ref
    ref[0] = bm[0]
    for k in range(1, bm.shape[0]):
        replace = bm[k] > ref[k - 1] + EXPCAST_TAU
        if invert is not None:
            replace = replace ^ np.asarray(invert[k], dtype=bool)
        ref[k] = np.where(replace, bm[k], ref[k - 1])
    return ref


# Margins of the rounding decisions. The oracle takes every decision of the
# low-bit path in fp64 on exact scores; a run that forms the scores with fp32
# accumulation (d products) and the code argument 8x + 104 with fp32 multiply-
# adds can take a decision that lies within rounding distance of its boundary
# the other way. The margin of a key's code argument (code units) is twice the
# worst case of: the accumulation, d * 2^-23 * sum_i |q_i k_i| for the key and
# for the reference's key, scaled by 8 * log2(e) / sqrt(d); the scale constant
# and the product with it, 2^-23 * |8x| and 2^-22 * |8m|; the bias 104 - 8m
# and the multiply-add, 2^-23 * 232. A replacement decision's margin (log2
# units) is the largest key margin of its block over 8.
def _fp8_margins(absdot, x, m, absdot_ref, c2, d):
    acc = d * 2.0 ** -23 * (absdot + absdot_ref[:, None]) * 8.0 * c2
    rnd = 2.0 ** -23 * np.abs(8.0 * x) + 2.0 ** -22 * np.abs(8.0 * m)[:, None] + 2.0 ** -23 * 232.0
    return 2.0 * (acc + rnd)


def attention_fp8(Qt, Kt, codes, mu, e, g: Geom, row_ptr, col_idx, blocks=None, invert=None,
                  diag=False):
    """Block-sparse attention with ExpCast-FP8 probabilities and V-Smooth
    values (readings above), row by row in col_idx order.

    Per selected block j of a row, on its real keys: x = q.k / sqrt(d) * log2(e),
    references m from ``expcast_reference`` over the blocks' row maxima,
    probabilities P = decode(expcast_code(x - m)), l_j = sum of P over the
    block; accumulators A += P @ (sigma * decode(codes_j)), L += l_j,
    M += l_j * mu_j, all rescaled together by 2^(m_old - m_new) when the
    reference moves. O = (A + M) / L, lse = ln(L) + (m - 6) * ln(2). Padding
    query slots: O = 0, lse = 0. Returns (Ot, lse) like ``attention``.

    ``invert``: {(b, h, i): bool [n, bs]} replacement decisions to take the
    other way in that mask row (``expcast_reference``).
    ``diag``: also return a dict of decision margins per query slot:
    ``flip_o`` [B,H,Npad,d] and ``flip_lse`` [B,H,Npad], bounds on how far O
    and lse move if every code whose argument lies within its margin of a
    rounding boundary (k + 1/2, k = 0..125) takes the neighbouring code (the
    probability moves by decode(k+1) - decode(k); O moves by that times
    |v - O| over L, lse by -ln(1 - sum |dP| / L)); ``thr_near`` [B,H,Npad]
    the number of replacement decisions within their margin of the threshold,
    and ``thr_first`` [B,H,Npad] the block position of the first (-1: none)."""
    Qt = np.asarray(Qt, dtype=np.float64)
    Kt = np.asarray(Kt, dtype=np.float64)
    B, H, Npad, d = Qt.shape
    nb, bs = g.nb, g.bs
    valid = slot_valid(g)
    Vr = e4m3_decode(codes) * np.exp2(np.asarray(e, dtype=np.float64))[:, :, None, None]
    Ot = np.full((B, H, Npad, d), np.nan)
    lse = np.full((B, H, Npad), np.nan)
    if diag:
        flip_o = np.zeros((B, H, Npad, d))
        flip_lse = np.zeros((B, H, Npad))
        thr_near = np.zeros((B, H, Npad), dtype=np.int64)
        thr_first = np.full((B, H, Npad), -1, dtype=np.int64)
    if blocks is None:
        blocks = [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    c2 = math.log2(math.e) / math.sqrt(d)
    for (b, h, i) in blocks:
        r = (b * H + h) * nb + i
        sel = np.asarray(col_idx[row_ptr[r]:row_ptr[r + 1]], dtype=np.int64)
        q_slots = np.arange(i * bs, (i + 1) * bs)
        q = Qt[b, h, q_slots]
        n_q = q.shape[0]
        keys = []
        xs = []
        for j in sel:
            ks = np.arange(j * bs, (j + 1) * bs)
            ks = ks[valid[ks]]
            keys.append(ks)
            xs.append((q @ Kt[b, h, ks].T) * c2)
        if len(sel):
            bmax = np.stack([x.max(axis=1) for x in xs])
            ref = expcast_reference(bmax, None if invert is None else invert.get((b, h, i)))
        m = np.full(n_q, -np.inf)
        A = np.zeros((n_q, d))
        L = np.zeros(n_q)
        M = np.zeros((n_q, d))
        F0 = np.zeros(n_q)       # sum of |dP| over near-boundary codes
        F1 = np.zeros((n_q, d))  # sum of |dP| |v|
        mkey = np.zeros(n_q)     # sum |q_i k_i| of the reference's key
        for idx, j in enumerate(sel):
            x = xs[idx]
            m_new = ref[idx]
            alpha = np.where(np.isfinite(m), np.exp2(np.where(np.isfinite(m), m - m_new, 0.0)), 0.0)
            A *= alpha[:, None]
            M *= alpha[:, None]
            L *= alpha
            F0 *= alpha
            F1 *= alpha[:, None]
            if diag:
                absdot = np.abs(q) @ np.abs(Kt[b, h, keys[idx]]).T
                moved = m_new != m
                arg = np.argmax(x, axis=1)
                mkey = np.where(moved, absdot[np.arange(n_q), arg], mkey)
                marg = _fp8_margins(absdot, x, m_new, mkey, c2, d)
                if idx > 0:
                    gap = np.abs(bmax[idx] - (m + EXPCAST_TAU))
                    near = gap <= marg.max(axis=1) / 8.0
                    rows = q_slots[near]
                    thr_first[b, h, rows] = np.where(thr_first[b, h, rows] < 0, idx,
                                                     thr_first[b, h, rows])
                    thr_near[b, h, q_slots] += near
            m = m_new
            y = 8.0 * (x - m[:, None]) + EXPCAST_BIAS
            P = e4m3_decode(expcast_code(x - m[:, None]))
            lj = P.sum(axis=1)
            vk = Vr[b, h, keys[idx]]
            A += P @ vk
            M += lj[:, None] * mu[b, h, j].astype(np.float64)[None, :]
            L += lj
            if diag:
                kb = np.floor(y - 0.5)  # boundary k + 1/2 just below y
                dist = np.minimum(np.abs(y - (kb + 0.5)), np.abs(y - (kb + 1.5)))
                kk = np.where(np.abs(y - (kb + 0.5)) <= np.abs(y - (kb + 1.5)), kb, kb + 1)
                hit = (dist <= marg) & (kk >= 0) & (kk <= 125)
                kc = np.clip(kk, 0, 125).astype(np.int64)
                dP = np.where(hit, e4m3_decode(kc + 1) - e4m3_decode(kc), 0.0)
                vd = np.abs(vk + mu[b, h, j].astype(np.float64)[None, :])
                F0 += dP.sum(axis=1)
                F1 += dP @ vd
        qv = valid[q_slots]
        with np.errstate(divide="ignore", invalid="ignore"):
            o = (A + M) / L[:, None]
            ls = np.log(L) + (m - (EXPCAST_BIAS - 56.0) / 8.0) * math.log(2.0)
            if diag:
                den = np.maximum(L - F0, 0.0)
                fo = np.where(F0[:, None] > 0, (F1 + np.abs(o) * F0[:, None]) / den[:, None], 0.0)
                fl = np.where(F0 > 0, -np.log(np.maximum(1.0 - F0 / L, 1e-300)), 0.0)
        o[~qv] = 0.0
        ls[~qv] = 0.0
        Ot[b, h, q_slots] = o
        lse[b, h, q_slots] = ls
        if diag:
            fo[~qv] = 0.0
            fl[~qv] = 0.0
            flip_o[b, h, q_slots] = fo
            flip_lse[b, h, q_slots] = fl
    if diag:
        return Ot, lse, {"flip_o": flip_o, "flip_lse": flip_lse, "thr_near": thr_near,
                         "thr_first": thr_first}
    return Ot, lse
