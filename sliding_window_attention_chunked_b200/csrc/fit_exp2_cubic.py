"""Fit the cubic behind the FMA-pipe exponential in exp2x2.cuh.

2^x is split as 2^n * 2^f with n the integer nearest x and f = x - n in [-1/2, 1/2]; 2^f is
taken from a cubic c0 + c1 f + c2 f^2 + c3 f^3. The coefficients minimise the largest relative
error over [-1/2, 1/2]. They are found with Lawson's algorithm (iteratively reweighted least
squares: each pass multiplies every grid point's weight by its current error, which drives the
weighted least-squares solution to the equal-ripple minimax one) on a grid of 20001 points, then
rounded to fp32. Run it to print the constants and their error; the kernel header holds its output.
"""
import numpy as np


def fit(grid=20001, passes=2000):
    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    V = np.vander(f, 4, increasing=True)
    w = np.full_like(f, 1.0 / grid)
    for _ in range(passes):
        s = np.sqrt(w)
        c = np.linalg.lstsq(V * (s / y)[:, None], s, rcond=None)[0]
        w = w * np.abs(V @ c / y - 1)
        w /= w.sum()
    return c.astype(np.float32)


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(np.polyval(c[::-1].astype(np.float64), f) / np.exp2(f) - 1).max()
    for i, x in enumerate(c):
        print(f"constexpr float kExpC{i} = {float(x)!r}f;")
    print(f"// largest relative error over [-1/2, 1/2]: {err:.3e}")
