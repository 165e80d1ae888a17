"""The identity the V-Smooth kernel's statistics pass relies on (VC-Attention:
Value Smoothing and Softmax Casting for Low-bit Attention, abstract: one scale
per head from the largest smoothed residual).

The kernel does not form every residual R = fl(v - mu) to find a block's
largest |R|: it keeps each channel's minimum and maximum and takes
max(fl(vmax - mu), fl(mu - vmin)) in fp32. That equals max_v |fl(v - mu)|
because round-to-nearest is monotone (v1 >= v2 implies fl(v1 - mu) >=
fl(v2 - mu)) and symmetric (|fl(x)| = fl(|x|)). Checked here in fp32 on
bf16-valued data: random blocks, constant blocks, zeros of both signs,
subnormals and wide exponent ranges."""
import numpy as np
import torch


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _cases(rng):
    yield _bf16(rng.standard_normal((128, 64)))
    yield _bf16(np.full((37, 64), 0.375))
    z = _bf16(rng.standard_normal((100, 64)))
    z[rng.random(z.shape) < 0.3] = 0.0
    z[rng.random(z.shape) < 0.3] = -0.0
    yield z
    t = _bf16(rng.standard_normal((64, 64)) * 1e-39)  # bf16 subnormals
    yield t
    w = _bf16(rng.standard_normal((128, 64)) * np.exp2(rng.integers(-60, 60, (128, 64))))
    yield w
    for _ in range(40):
        n = int(rng.integers(1, 129))
        s = np.exp2(rng.integers(-30, 30))
        yield _bf16(rng.standard_normal((n, 64)) * s + rng.standard_normal() * s * 100)


def test_block_max_residual_from_channel_extremes():
    rng = np.random.default_rng(3)
    for v in _cases(rng):
        mu = (v.astype(np.float64).sum(axis=0) / v.shape[0]).astype(np.float32)
        direct = np.abs(v - mu[None, :]).max(axis=0)          # fp32 residuals
        vmax, vmin = v.max(axis=0), v.min(axis=0)
        ext = np.maximum(np.float32(0.0), np.maximum(vmax - mu, mu - vmin))  # fp32
        assert direct.dtype == np.float32 and ext.dtype == np.float32
        assert np.array_equal(direct, ext)
