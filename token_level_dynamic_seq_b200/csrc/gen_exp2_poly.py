"""Derive the coefficients of the polynomial exp2 used in the softmax.

Method (Cody-Waite style range reduction + minimax polynomial): for x <= 8,
write x = n + f with n = round(x) and f in [-1/2, 1/2]; then 2^x = 2^n * p(f),
where p is the degree-3 polynomial minimising the maximum RELATIVE error
|p(f) / 2^f - 1| on [-1/2, 1/2].  The minimax fit is computed here with the
Remez exchange algorithm (equioscillation on 5 reference points), from the
mathematics of 2^f alone.  2^n is applied by adding n to the exponent field.

Running this script prints the coefficients in float32 hex and decimal, as
they appear in ptx.cuh (exp2_poly), and the achieved relative error.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}
        A = np.zeros((n, n))
        b = np.exp2(x)
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(A, b)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extrema of err between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        # keep the n alternating extrema with the largest magnitudes
        cand = idx[np.argsort(-np.abs(err[idx]))]
        chosen = []
        for i in cand:
            if all(abs(i - j) > 100 for j in chosen):
                chosen.append(i)
            if len(chosen) == n:
                break
        x = grid[np.sort(np.array(chosen))]
    return c, np.max(np.abs(err))


def f32_hex(v):
    return "0x%08x" % np.float32(v).view(np.uint32)


if __name__ == "__main__":
    c, e = remez()
    c32 = np.float32(c)
    f = np.linspace(LO, HI, 100001).astype(np.float32)
    p = ((c32[3] * f + c32[2]) * f + c32[1]) * f + c32[0]
    e32 = np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0))
    for i, v in enumerate(c32):
        print(f"c{i} = {f32_hex(v)}  # {float(v):.9g}")
    print(f"max relative error: {e:.3e} (double), {e32:.3e} (float32 Horner)")
