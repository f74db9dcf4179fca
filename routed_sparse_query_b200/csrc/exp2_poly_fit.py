"""Fits the polynomial exp2 used by the attention softmax on the FMA pipe.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by a degree-3 polynomial p(f) with minimax relative error,
found by the Remez exchange algorithm (E. Remez, 1934; see e.g. Muller,
"Elementary Functions: Algorithms and Implementation", ch. 3): solve
p(x_i) - 2^x_i = (-1)^i E 2^x_i on d+2 reference points, move the points to
the extrema of the weighted error, repeat. All four coefficients are free
(pinning p(0) = 1 would raise the error about six-fold; the values are
rounded to bf16 afterwards, where 1 - 7.5e-5 rounds to 1).

Run: python exp2_poly_fit.py  -> prints the coefficients as fp32 literals and
the maximum relative error over [-1/2, 1/2] evaluated in fp32 Horner form.
"""
import numpy as np


def remez(deg=3, a=-0.5, b=0.5, iters=30, fix_c0=False):
    f = lambda x: np.exp2(x)
    n_free = deg if fix_c0 else deg + 1
    k = n_free + 1  # reference points
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(k)[::-1] / (k - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # unknowns: free coefficients and E
        A = np.zeros((k, k))
        rhs = np.zeros(k)
        for i, xi in enumerate(x):
            col = 0
            for p in range(0 if not fix_c0 else 1, deg + 1):
                A[i, col] = xi ** p
                col += 1
            A[i, -1] = -((-1) ** i) * f(xi)
            rhs[i] = f(xi) - (1.0 if fix_c0 else 0.0)
        sol = np.linalg.solve(A, rhs)
        c = ([1.0] if fix_c0 else []) + list(sol[:-1])
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of err between sign changes
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        cand = sorted(idx, key=lambda j: -abs(err[j]))
        pts = sorted(cand[:k])
        if len(pts) == k:
            x = grid[pts]
    return np.array(c), np.abs(err).max()


def fp32_horner_error(c):
    x = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    c32 = c.astype(np.float32)
    p = np.full_like(x, c32[3])
    for q in (2, 1, 0):
        p = (p * x + c32[q]).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c, e = remez()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}f" for v in c.astype(np.float32)))
    print(f"minimax relative error {e:.3e}; fp32 Horner max relative error {fp32_horner_error(c):.3e}")
