"""Fits the cubic p(f) ~ 2^f on [-1/2, 1/2] used by the kernels' FMA-pipe exp2.

Method (Cody-Waite style argument split): 2^x = 2^n * 2^f with n = round(x)
and f = x - n in [-1/2, 1/2]. n is obtained with one fp32 add of 1.5 * 2^23
(which leaves round(x) in the low mantissa bits), 2^f by the cubic below, and
2^n by adding n to the fp32 exponent field. The cubic minimises the maximum
relative error p(f) / 2^f - 1 over [-1/2, 1/2] (Remez exchange). Run this file
to print the coefficients the kernels use and their error bound; the CPU test
test_exp2_poly.py re-derives them and checks the bound in fp32 arithmetic.
"""
import numpy as np

LO, HI = -0.5, 0.5


def fit(degree: int = 3, iters: int = 40):
    n = degree + 2                                  # deg + 1 coefficients + levelled error
    xs = (LO + HI) / 2 - (HI - LO) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(LO, HI, 400001)
    for _ in range(iters):
        a = np.zeros((n, n))
        for i, x in enumerate(xs):
            t = 2.0 ** x
            a[i, :degree + 1] = [x ** k / t for k in range(degree + 1)]
            a[i, degree + 1] = -((-1) ** i)
        sol = np.linalg.solve(a, np.ones(n))
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1
        # exchange: one extremum of |err| per alternating interval
        bounds = np.r_[LO, (xs[:-1] + xs[1:]) / 2, HI]
        new = []
        for lo, hi in zip(bounds[:-1], bounds[1:]):
            sel = np.where((grid >= lo) & (grid <= hi))[0]
            new.append(grid[sel[np.argmax(np.abs(err[sel]))]])
        xs = np.array(new)
    return c, float(np.abs(err).max())


def coefficients_f32():
    c, _ = fit()
    return [float(np.float32(v)) for v in c]


if __name__ == "__main__":
    c, e = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print("fp32 constants:", ", ".join(repr(v) for v in coefficients_f32()))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
