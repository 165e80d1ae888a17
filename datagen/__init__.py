"""Seeded synthetic Q/K/V for the five workloads of the block-sparse attention path.

This module only makes inputs. It holds none of the method's arithmetic
(no permutation, pooling, scoring, selection or attention), so both the fp64
oracle and the CUDA path may consume its output: they receive identical bits.

The inputs stand in for video-DiT layer activations (the pages evaluate on
Wan and HunyuanVideo with VBench prompts, none of which are available here).
Recipe, per head (FVAttn abstract: video DiT self-attention over a
spatio-temporal latent grid):

* every channel c of a latent field X has eight plane-wave modes,
  ``X[n, c] = sum_m a[c,m] * cos(2*pi * f[c,m] . (t_n, h_n, w_n) + phi[c,m])
  + 0.3 * eps[n, c]`` with ``a ~ N(0,1)``, ``f ~ U[0, 0.25]^3``,
  ``phi ~ U[0, 2*pi)``, ``eps ~ N(0,1)``;
* ``Q = X Wq``, ``K = X Wk`` with ``Wq, Wk ~ N(0, 1/d)`` (d x d), ``V ~ N(0,1)``;
* for the bf16 workloads a 3-D rotary embedding acts on Q and K: the head
  dimension is split into t/h/w segments, each segment rotates interleaved
  pairs ``(2i, 2i+1)`` by ``coord * 10000**(-2i/s)`` where s is the segment width;
* the "stress" workload scales every mode amplitude of head h by
  ``s_h ~ U[0.2, 3]`` (noise unscaled) and gives head h the Top-p value
  ``(0.5, 0.7, 0.9, 0.97, 0.99)[h % 5]``.

All draws come from ``numpy.random.default_rng(seed)`` in a fixed order:
stress scales first (stress only), then per head ``a, f, phi, eps, Wq, Wk, V``
(the tiny workload draws ``a, f, phi, eps`` once, shared by its heads, then
per head ``Wq, Wk, V``). Fields are evaluated in fp64 (on the given torch
device, for speed) and rounded once to the workload dtype.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and routing parameters of one synthetic workload."""

    name: str
    B: int
    H: int
    T: int
    Hh: int
    W: int
    d: int
    cube: tuple  # (ct, ch, cw)
    dtype: str  # "f32" or "bf16"
    top_p: tuple  # per head (len H) or a single value
    top_k: int
    rope_split: Optional[tuple] = None  # (t, h, w) widths, sum = d
    per_head_modes: bool = True
    amp_range: Optional[tuple] = None  # (lo, hi) for per-head amplitude scale
    order: str = "cube"  # block organisation the layer is run with ("cube" / "hilbert")

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.W

    def top_p_per_head(self) -> list:
        if len(self.top_p) == 1:
            return [float(self.top_p[0])] * self.H
        return [float(self.top_p[h % len(self.top_p)]) for h in range(self.H)]

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


STRESS_P = (0.5, 0.7, 0.9, 0.97, 0.99)

WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 4, 8, 8, 64, (4, 4, 4), "f32", (0.9,), 1,
                     rope_split=None, per_head_modes=False),
    "small": Workload("small", 1, 8, 8, 16, 16, 64, (4, 4, 4), "bf16", (0.9,), 4,
                      rope_split=(16, 24, 24)),
    "wan": Workload("wan", 1, 40, 21, 30, 52, 128, (2, 8, 8), "bf16", (0.9,), 8,
                    rope_split=(44, 42, 42)),
    "hunyuan": Workload("hunyuan", 1, 24, 33, 45, 80, 128, (2, 8, 8), "bf16", (0.85,), 8,
                        rope_split=(44, 42, 42)),
    "stress": Workload("stress", 1, 40, 21, 30, 52, 128, (2, 8, 8), "bf16", STRESS_P, 8,
                       rope_split=(44, 42, 42), amp_range=(0.2, 3.0)),
    # the Wan layer cut to 8 heads: same kernels and tile shapes, 0.24 GB of
    # reordered q/k/v (still larger than L2), used for profiler captures
    "wan8": Workload("wan8", 1, 8, 21, 30, 52, 128, (2, 8, 8), "bf16", (0.9,), 8,
                     rope_split=(44, 42, 42)),
    # the stress recipe on 10 heads (each Top-p value twice), for profiler
    # captures of the two schedules
    "stress10": Workload("stress10", 1, 10, 21, 30, 52, 128, (2, 8, 8), "bf16", STRESS_P, 8,
                         rope_split=(44, 42, 42), amp_range=(0.2, 3.0)),
}


def custom(name: str, B: int, H: int, T: int, Hh: int, W: int, d: int, cube, dtype="bf16",
           top_p=(0.9,), top_k=4, rope_split=None, per_head_modes=True, amp_range=None,
           order="cube") -> Workload:
    """A workload of any shape, built with the same recipe (used for ragged/edge tests)."""
    return Workload(name, B, H, T, Hh, W, d, tuple(cube), dtype, tuple(top_p), top_k,
                    rope_split, per_head_modes, amp_range, order)


def with_order(wl: Workload, order: str) -> Workload:
    """The same inputs run with another block organisation."""
    return dataclasses.replace(wl, name=f"{wl.name}_{order}", order=order)


def _coords(T: int, Hh: int, W: int):
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.float64)  # [N,3]


def _draw_modes(rng, d):
    a = rng.standard_normal((d, 8))
    f = rng.uniform(0.0, 0.25, size=(d, 8, 3))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=(d, 8))
    return a, f, phi


def _field(coords_t, a, f, phi, eps, scale, device):
    """X[n,c] = scale * sum_m a cos(2 pi f.x + phi) + 0.3 eps, evaluated in fp64."""
    N = coords_t.shape[0]
    d = a.shape[0]
    a_t = torch.from_numpy(a * scale).to(device)
    f_t = torch.from_numpy(f).to(device)
    phi_t = torch.from_numpy(phi).to(device)
    X = torch.empty((N, d), dtype=torch.float64, device=device)
    chunk = max(1, (1 << 24) // (d * 8))
    for s in range(0, N, chunk):
        x = coords_t[s:s + chunk]  # [n,3]
        ph = 2.0 * math.pi * torch.einsum("nk,cmk->ncm", x, f_t) + phi_t  # [n,d,8]
        X[s:s + chunk] = (torch.cos(ph) * a_t).sum(-1)
    X += 0.3 * torch.from_numpy(eps).to(device)
    return X


def _rope(Y, coords_t, split):
    """Interleaved-pair 3-D rotary embedding over (t, h, w) segments, base 10000."""
    out = Y.clone()
    off = 0
    for axis, s in enumerate(split):
        half = s // 2
        i = torch.arange(half, dtype=torch.float64, device=Y.device)
        theta = torch.pow(torch.tensor(10000.0, dtype=torch.float64, device=Y.device), -2.0 * i / s)
        ang = coords_t[:, axis:axis + 1] * theta[None, :]  # [N, half]
        c, sn = torch.cos(ang), torch.sin(ang)
        x0 = Y[:, off:off + 2 * half:2]
        x1 = Y[:, off + 1:off + 2 * half:2]
        out[:, off:off + 2 * half:2] = x0 * c - x1 * sn
        out[:, off + 1:off + 2 * half:2] = x0 * sn + x1 * c
        off += s
    return out


def generate(wl: Workload, seed: int = 0, device: str | torch.device = "cpu",
             out_device: str | torch.device | None = None):
    """Return (q, k, v) as contiguous ``[B, H, N, d]`` tensors of the workload dtype.

    ``device`` is where the fp64 fields are evaluated; ``out_device`` where the
    rounded tensors are returned (defaults to ``device``).
    """
    out_device = device if out_device is None else out_device
    rng = np.random.default_rng(seed)
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    dt = wl.torch_dtype
    q = torch.empty((B, H, N, d), dtype=dt, device=out_device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    coords_t = torch.from_numpy(_coords(wl.T, wl.Hh, wl.W)).to(device)
    scales = None
    if wl.amp_range is not None:
        scales = rng.uniform(wl.amp_range[0], wl.amp_range[1], size=(B, H))
    shared = None
    if not wl.per_head_modes:
        a, f, phi = _draw_modes(rng, d)
        eps = rng.standard_normal((N, d))
        shared = (a, f, phi, eps)
    for b in range(B):
        for h in range(H):
            if shared is None:
                a, f, phi = _draw_modes(rng, d)
                eps = rng.standard_normal((N, d))
            else:
                a, f, phi, eps = shared
            wq = rng.standard_normal((d, d)) / math.sqrt(d)
            wk = rng.standard_normal((d, d)) / math.sqrt(d)
            vv = rng.standard_normal((N, d))
            scale = 1.0 if scales is None else float(scales[b, h])
            X = _field(coords_t, a, f, phi, eps, scale, device)
            Q = X @ torch.from_numpy(wq).to(device)
            K = X @ torch.from_numpy(wk).to(device)
            if wl.rope_split is not None:
                Q = _rope(Q, coords_t, wl.rope_split)
                K = _rope(K, coords_t, wl.rope_split)
            q[b, h] = Q.to(dt).to(out_device)
            k[b, h] = K.to(dt).to(out_device)
            v[b, h] = torch.from_numpy(vv).to(device).to(dt).to(out_device)
    return q, k, v


def random_qkv(B: int, H: int, N: int, d: int, dtype=torch.bfloat16, seed: int = 0,
               device="cpu"):
    """Plain N(0,1) inputs for edge-case tests (no structure)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        x = rng.standard_normal((B, H, N, d))
        out.append(torch.from_numpy(x).to(dtype).to(device))
    return tuple(out)


__all__ = ["Workload", "WORKLOADS", "STRESS_P", "custom", "generate", "random_qkv", "with_order"]
