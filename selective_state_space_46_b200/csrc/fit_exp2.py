"""Coefficients of the FP32-pipe exp2 in scan.cuh (exp2_fma2).

2^f on [-1/2, 1/2] by p(f) = 1 + f q(f) with q of degree 4: the constant term is exactly 1, so
the error vanishes as f -> 0 and decay factors close to 1 (the long-memory states, whose
errors compound over many steps) carry no systematic bias.  q minimises the maximum relative
error of p, |p(f) - 2^f| / 2^f = |f| / 2^f * |q(f) - (2^f - 1) / f|, made equi-oscillating with
Lawson's iteratively reweighted least squares on Chebyshev points, in fp64; the coefficients
are then rounded to fp32.  Run it to print the constants; the CPU tests re-run the fit and
check that the header holds these values and that the fp32 Horner evaluation with the range
reduction stays within the stated bounds.
"""
import numpy as np

DEGREE = 5
ITERATIONS = 40
POINTS = 4001


def fit(degree: int = DEGREE) -> np.ndarray:
    f = np.cos(np.linspace(0.0, np.pi, POINTS)) * 0.5
    f = f[np.abs(f) > 1e-12]
    y = np.exp2(f)
    target = np.expm1(f * np.log(2.0)) / f       # (2^f - 1) / f
    vander = np.vander(f, degree, increasing=True)
    scale = np.abs(f) / y                        # relative error of p per unit error of q
    weight = np.ones_like(f)
    coef = None
    for _ in range(ITERATIONS):
        w = np.sqrt(weight) * scale
        coef, *_ = np.linalg.lstsq(vander * w[:, None], target * w, rcond=None)
        err = np.abs(vander @ coef - target) * scale
        weight = weight * err
        weight /= weight.sum()
    return np.concatenate([[1.0], coef]).astype(np.float32)


if __name__ == "__main__":
    for k, c in enumerate(fit()):
        print(f"constexpr float kExp2C{k} = {float(c)!r}f;")
