"""Fits the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the FMA-pipe exp2 in
the attention kernel, and prints it as C constants.

Method (written for this library): minimise the maximum *relative* error
|p(f) / 2^f - 1| over [-1/2, 1/2] with a degree-4 polynomial, by the Remez
exchange algorithm started from Chebyshev nodes, in float64; the coefficients
are then rounded to float32 and the error is re-measured on a dense grid with
float32 Horner evaluation.  Run: python gen_exp2_poly.py
"""
import numpy as np

DEG = 4
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i   (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new extrema: one per sign-alternating segment
        sign = np.sign(err)
        idx = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sign[i] != sign[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = i
        idx = np.array(idx)
        if len(idx) > n:
            # keep the n largest, preserving alternation order
            keep = np.sort(np.argsort(-np.abs(err[idx]))[:n])
            idx = idx[keep]
        if len(idx) == n:
            x = grid[idx]
    return c


def f32_horner_error(c32):
    f = np.linspace(LO, HI, 400001).astype(np.float32)
    acc = np.float32(c32[-1]) * np.ones_like(f)
    for a in c32[-2::-1]:
        acc = (acc * f + np.float32(a)).astype(np.float32)
    return float(np.max(np.abs(acc.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    c = remez()
    c32 = c.astype(np.float32)
    print(f"// degree-{DEG} minimax (relative) fit of 2^f on [-1/2, 1/2]; "
          f"max rel error {f32_horner_error(c32):.3e} with float32 Horner")
    for i, a in enumerate(c32):
        print(f"constexpr float EXP2_C{i} = {float(a):.9e}f;")
