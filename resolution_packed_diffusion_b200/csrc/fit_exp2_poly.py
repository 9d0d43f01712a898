"""Coefficients of the polynomial 2^f, f in [-1/2, 1/2], used by exp2_poly()
in mf_ptx.cuh.

Method: Remez exchange for the minimax *relative* error of a degree-3
polynomial p(f) ~ 2^f (E. Remez, 1934; any numerical analysis text). The
kernel reduces 2^x to 2^j * 2^f with j = round(x) (Cody-Waite style range
reduction with a single exact step, since j is an integer and f = x - j is
exact in float32), so the polynomial only has to cover [-1/2, 1/2].

    python resolution_packed_diffusion_b200/csrc/fit_exp2_poly.py

prints the float32 coefficients c0..c3 and the maximum relative error of the
float32 Horner evaluation over a dense grid (about 7.5e-5, far below the 2^-9
relative rounding of the bf16 probabilities the kernel stores).
"""

import numpy as np


def remez_exp2(deg=3, lo=-0.5, hi=0.5, iters=40):
    n = deg + 2
    k = np.arange(n)
    xs = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 400001)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i (1 + (-1)^i E) = 0 for the n reference points
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = xs[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xs[i]
        sol = np.linalg.solve(A, 2.0 ** xs)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        turn = np.where(np.diff(np.sign(np.diff(err))) != 0)[0] + 1
        cand = grid[np.concatenate([[0], turn, [len(grid) - 1]])]
        if len(cand) == n:
            xs = cand
        else:
            e = np.abs(np.polyval(c[::-1], cand) / 2.0 ** cand - 1.0)
            xs = np.sort(cand[np.argsort(-e)[:n]])
    return c


def horner_f32(c, f):
    p = np.float32(c[-1])
    for cc in c[-2::-1]:
        p = (p * f + np.float32(cc)).astype(np.float32)
    return p


if __name__ == "__main__":
    c = remez_exp2().astype(np.float32)
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    err = np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0).max()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v):.9e}f")
    print(f"max relative error (float32 Horner) = {err:.3e}")
