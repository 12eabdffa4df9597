"""Fit the polynomial the attention kernel uses to evaluate 2^f on the FMA
pipe, f in [-1/2, 1/2] (after Cody-Waite range reduction 2^x = 2^n * 2^f,
n = round(x)).

Method: Remez exchange for the minimax *relative* error of a degree-D
polynomial p(f) ~ 2^f, then rounding of the coefficients to binary32 and a
dense re-evaluation (in binary64, Horner with binary32 coefficients) of the
resulting relative error.  Prints the coefficients as C literals.

Usage: python -m quantized_fp8_attention_b200.tools.fit_exp2_poly [degree]
"""

import sys

import numpy as np


def remez_relative(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.flatnonzero(np.diff(s) != 0)
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) < n:
            break
        # keep n alternating points with the largest errors
        ext = np.array(ext)
        while len(ext) > n:
            # drop the smaller end
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[ext]
    return c


def evaluate(c32, lo=-0.5, hi=0.5):
    g = np.linspace(lo, hi, 2000001)
    acc = np.full_like(g, c32[-1], dtype=np.float64)
    for ci in c32[-2::-1]:
        acc = acc * g + ci
    return float(np.max(np.abs(acc / np.exp2(g) - 1.0)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c = remez_relative(deg)
    c32 = np.array(c, dtype=np.float32).astype(np.float64)
    print(f"// degree {deg}, max relative error (binary64 Horner, binary32 coefficients): {evaluate(c32):.3e}")
    for i, ci in enumerate(np.array(c, dtype=np.float32)):
        print(f"constexpr float kExp2C{i} = {float(ci)!r}f;  // {ci.view(np.uint32):#010x}")


if __name__ == "__main__":
    main()
