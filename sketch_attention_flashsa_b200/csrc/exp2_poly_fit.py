"""Fits the polynomial behind the FMA-pipe exp2 of the SA kernels.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in [-1/2, 1/2]; p is the
degree-3 polynomial minimising the maximum RELATIVE error |p(f) / 2^f - 1| on that interval,
found with the Remez exchange algorithm (equioscillation at degree + 2 = 5 points). The
constants printed here are the ones hard-coded in sa_proto_fwd.cu; rerun this script to check
them:  python sketch_attention_flashsa_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=40):
    f = lambda x: np.exp2(x)  # noqa: E731
    n = deg + 2
    # Chebyshev points as the first reference
    k = np.arange(n)
    xs = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve  sum_j c_j x_i^j + (-1)^i E f(x_i) = f(x_i)   (relative error weight 1/f)
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1.0
        # new reference: extrema of the error, one per sign change segment
        sign = np.sign(err)
        idx = []
        start = 0
        for j in range(1, len(grid)):
            if sign[j] != sign[j - 1]:
                seg = slice(start, j)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = j
        idx.append(start + int(np.argmax(np.abs(err[start:]))))
        if len(idx) != n:
            break
        xs = grid[idx]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 100001)
    e32 = np.abs(np.polyval(c32.astype(np.float64)[::-1], grid) / np.exp2(grid) - 1).max()
    print("coefficients c0..c3 (float32):", [float(x) for x in c32])
    print("hex:", [hex(np.float32(x).view(np.uint32)) for x in c32])
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32 coefficients)")
