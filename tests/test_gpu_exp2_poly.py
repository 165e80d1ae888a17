"""The attention softmax takes one exponential pair in eight on the FMA pipe
(exp2_poly2: round-to-nearest range reduction, a degree-3 minimax polynomial
for 2^f on [-1/2, 1/2], the integer part added to the exponent field). Its
error bound: the fp32 polynomial is within 7.48e-5 relative of 2^f
(block_sparse_attention_sba_b200/csrc/fit_exp2_poly.py evaluates it on a fine
grid); the reduction (f = x - round(x)) and the exponent add are exact for
results in the normal range. So on [-125, 0] the result is within 8e-5
relative of the exact 2^x; below -125 the input is clamped to -125."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_exp2_poly_within_its_bound_of_exact_exp2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_sba_b200 as sba
    g = torch.Generator().manual_seed(0)
    parts = [torch.linspace(-125.0, 0.0, 4_000_001),
             -125.0 * torch.rand(1_000_000, generator=g),
             torch.arange(-125, 1, dtype=torch.float32),            # integers: f = 0
             torch.arange(-125, 0, dtype=torch.float32) + 0.5,      # ties of the reduction
             torch.arange(-125, 0, dtype=torch.float32) + 0.4999999,
             torch.tensor([-124.99999, -1e-7, -0.0, 0.0])]
    x = torch.cat(parts).float()
    y = torch.empty_like(x, device="cuda")
    sba.sba_debug_exp2_poly(x.cuda(), y)
    torch.cuda.synchronize()
    got = y.cpu().double().numpy()
    exact = np.exp2(x.double().numpy())
    rel = np.abs(got / exact - 1.0)
    assert rel.max() <= 8e-5, (float(rel.max()), float(x[int(np.argmax(rel))]))
    # at integers f = 0, so the result is the polynomial's constant term
    # times 2^x exactly
    k = torch.arange(-125, 1, dtype=torch.float32, device="cuda")
    yk = torch.empty_like(k)
    sba.sba_debug_exp2_poly(k, yk)
    torch.cuda.synchronize()
    c0 = float(np.float32(0.99992806))
    assert np.array_equal(yk.cpu().double().numpy(), c0 * np.exp2(k.cpu().double().numpy()))
    # clamped to -125 below it (so the result is c0 * 2^-125); odd length handled
    z = torch.tensor([-130.0, -1000.0, -float("inf")], device="cuda")
    w = torch.empty_like(z)
    sba.sba_debug_exp2_poly(z, w)
    torch.cuda.synchronize()
    assert np.all(w.cpu().double().numpy() == c0 * 2.0 ** -125)
