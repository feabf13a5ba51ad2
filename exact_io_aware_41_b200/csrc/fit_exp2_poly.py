"""Fits the polynomial behind the FMA-pipe exp2 used by the prefill softmax.

Range reduction after Cody and Waite ("Software Manual for the Elementary Functions", 1980):
2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]. On that interval 2^f is
approximated by p(f) = c0 + c1 f + c2 f^2 + c3 f^3, evaluated by Horner's rule (three FMAs), with
coefficients chosen by a Remez exchange so that the relative error p(f) / 2^f - 1 equi-oscillates
(minimax in the relative sense). The printed fp32 coefficients are the ones compiled into
attn_fwd.cu; the fit reaches a maximum relative error of about 7.5e-5, well below the 2^-9
relative rounding of the bf16 probabilities the tensor cores consume.

Run: python exact_io_aware_41_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(degree: int = 3, iters: int = 60, lo: float = -0.5, hi: float = 0.5):
    n = degree + 1                       # coefficients c0..c_degree
    k = np.arange(n + 1)
    ref = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / n)  # Chebyshev extrema
    grid = np.linspace(lo, hi, 400001)

    def rel_err(c, f):
        return sum(c[j] * f ** j for j in range(n)) / 2.0 ** f - 1.0

    c = None
    for _ in range(iters):
        # p(f_i) = 2^f_i * (1 + (-1)^i E) at the n + 1 reference points: a linear system in (c, E)
        t = 2.0 ** ref
        A = np.zeros((n + 1, n + 1))
        for j in range(n):
            A[:, j] = ref ** j
        A[:, n] = -((-1.0) ** np.arange(n + 1)) * t
        c = np.linalg.solve(A, t)[:n]
        err = rel_err(c, grid)
        # exchange: the extremum of |err| on each run of constant sign
        sgn = np.sign(err)
        idx, start = [], 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sgn[i] != sgn[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = i
        if len(idx) != n + 1:
            break
        ref = grid[np.array(idx)]
    return c, float(np.abs(rel_err(c, grid)).max())


if __name__ == "__main__":
    c, e = fit(3)
    for j, cj in enumerate(c):
        print(f"c{j} = {float(np.float32(cj))!r:>14}f   ({cj:.17g})")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
