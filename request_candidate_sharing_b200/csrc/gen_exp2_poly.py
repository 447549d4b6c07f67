"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2] used by the
attention softmax for the share of its exponentials computed on the FMA pipe.

Method: minimax fit of the RELATIVE error by the Remez exchange algorithm (E. Ya. Remez, 1934; see
J.-M. Muller, "Elementary Functions: Algorithms and Implementation", ch. 3).  The argument is
reduced as x = n + f with n = round-to-nearest(x) obtained by adding and subtracting 1.5 * 2^23
(Muller, ch. 11, "shift" trick), so f lies in [-1/2, 1/2] and 2^x = 2^n * 2^f, with 2^n applied by
adding n to the exponent field.

    python gen_exp2_poly.py        # prints the float32 coefficients and the max relative error
"""
import numpy as np


def remez(n: int, iters: int = 30):
    a, b = -0.5, 0.5
    k = np.arange(n + 2)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the n + 2 reference points
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, :n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** xi
        c = np.linalg.solve(A, 2.0 ** x)[:n + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        cuts = np.concatenate(([0], np.where(np.diff(np.sign(err)) != 0)[0] + 1, [grid.size]))
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(cuts[:-1], cuts[1:])]
        if len(ext) == n + 2:
            x = grid[ext]
    return c.astype(np.float32), float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez(3)
    print("coefficients (c0..c3):", ", ".join(f"{float(v):.9g}f" for v in c))
    print("max relative error:", e)
