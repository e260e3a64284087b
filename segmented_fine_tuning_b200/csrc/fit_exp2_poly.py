"""Derives the coefficients of the cubic that the attention kernels use for
part of their 2^x evaluations (the rest go to the hardware ex2 unit).

Method: range reduction x = n + f with n = round(x), f in [-1/2, 1/2], and
2^x = 2^n * p(f), where p is the degree-3 polynomial of least maximum
relative error to 2^f on [-1/2, 1/2].  The minimax fit is found with
Lawson's algorithm (iteratively reweighted least squares; C. L. Lawson,
"Contributions to the theory of linear least maximum approximation", 1961):
each pass solves a weighted least-squares problem on a dense grid and
multiplies every weight by that point's current error.

Run as a script to print the coefficients as C hex-float literals; the test
suite calls fit() to check the constants compiled into the kernels and the
error bound they reach in fp32 Horner evaluation.
"""
import numpy as np

DEGREE = 3


def fit(degree=DEGREE, points=4001, passes=400):
    f = np.linspace(-0.5, 0.5, points)
    target = np.exp2(f)
    # relative error p(f)/2^f - 1 is linear in the coefficients: rows f^k / 2^f
    A = np.stack([f ** k for k in range(degree + 1)], axis=1) / target[:, None]
    w = np.full(points, 1.0 / points)
    c = None
    for _ in range(passes):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        err = np.abs(A @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c, float(np.max(np.abs(A @ c - 1.0)))


if __name__ == "__main__":
    c, e = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(np.float32(v)).hex()}f  // {v:.9g}")
    print(f"max relative error (fp64 evaluation): {e:.3e}")
