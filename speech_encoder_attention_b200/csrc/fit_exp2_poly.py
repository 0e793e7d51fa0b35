"""Fits the cubic used for 2^f, f in [-1/2, 1/2], in the software exp2 of the
attention softmax (flash_attn.cuh).

Method: Remez exchange for the minimax *relative* error of a degree-3
polynomial c0 + c1 f + c2 f^2 + c3 f^3 against 2^f, started from Chebyshev
nodes, then the coefficients are rounded to fp32 and the error re-measured on
a dense grid. Printing the result is all this script does:

    python speech_encoder_attention_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def remez(deg=3, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve sum_j c_j x_i^j + (-1)^i E f(x_i) = f(x_i)  (relative error weight 1/f)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep the n largest alternating extrema
        while len(idx) > n:
            drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
            idx.pop(drop)
        x = grid[idx]
    return c


def main():
    c = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 400001)
    approx = np.polyval(c32.astype(np.float64)[::-1], grid)
    rel = np.abs(approx - np.exp2(grid)) / np.exp2(grid)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r:>24}  ({ci.view(np.uint32):#010x})")
    print(f"max relative error {rel.max():.3e} ({rel.max() / 2**-11:.3f} of an fp16 half-ulp)")


if __name__ == "__main__":
    main()
