"""Coefficients of exp2_poly2 (ptx.cuh): the degree-3 polynomial p(f) ~ 2^f on
f in [-1/2, 1/2] with the smallest maximum relative error |p(f) / 2^f - 1|.

Method: the Remez exchange algorithm for a weighted minimax fit (weight
2^-f, i.e. relative error). Start from the Chebyshev extrema; at each step
solve p(x_i) - 2^(x_i) = (-1)^i E 2^(x_i) at the deg+2 reference points for
the coefficients and the levelled error E, then move each reference point to
the extremum of the error on its sign-alternation interval. It converges when
the reference no longer moves; the levelled error is then the maximum.

Run: python fit_exp2_poly.py   (prints the fp32 coefficients, highest degree
first, and the maximum relative error of the fp32 polynomial on a fine grid).
"""
import numpy as np


def remez_exp2(deg: int = 3, iters: int = 50, grid: int = 400001):
    m = deg + 2
    x = 0.5 * np.cos(np.pi * np.arange(m) / (m - 1))[::-1]
    t = np.linspace(-0.5, 0.5, grid)
    c = None
    for _ in range(iters):
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        e = np.polyval(c[::-1], t) / np.exp2(t) - 1.0
        cuts = [0] + list(np.nonzero(np.diff(np.sign(e)) != 0)[0] + 1) + [grid]
        new = np.array([t[a + int(np.argmax(np.abs(e[a:b])))] for a, b in zip(cuts[:-1], cuts[1:])])
        if new.size != m or np.allclose(new, x, atol=1e-12):
            break
        x = new
    return c  # lowest degree first


def main():
    c = remez_exp2()
    c32 = c.astype(np.float32)
    t = np.linspace(-0.5, 0.5, 400001)
    # evaluate the fp32 Horner scheme the kernel uses
    f = t.astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * f + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    print("coefficients (f^3, f^2, f^1, f^0):", ", ".join(f"{float(v):.8g}f" for v in c32[::-1]))
    print(f"max relative error in fp32: {rel.max():.3g}")


if __name__ == "__main__":
    main()
