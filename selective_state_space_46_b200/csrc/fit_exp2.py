"""Coefficients of the FP32-pipe exp2 in device_common.cuh (exp2_fma2).

2^f on [-1/2, 1/2] by a degree-5 polynomial whose relative error is made equi-oscillating
(minimax) with Lawson's iteratively reweighted least squares on Chebyshev points, in fp64;
the coefficients are then rounded to fp32.  Run it to print the constants; the CPU tests
re-run the fit and check that the header holds these values and that the fp32 Horner
evaluation with the range reduction stays within the stated bound.
"""
import numpy as np

DEGREE = 5
ITERATIONS = 30
POINTS = 4000


def fit(degree: int = DEGREE) -> np.ndarray:
    f = np.cos(np.linspace(0.0, np.pi, POINTS)) * 0.5
    y = np.exp2(f)
    vander = np.vander(f, degree + 1, increasing=True)
    weight = np.ones_like(f)
    coef = None
    for _ in range(ITERATIONS):
        w = weight / y
        coef, *_ = np.linalg.lstsq(vander * w[:, None], y * w, rcond=None)
        err = np.abs(vander @ coef - y) / y
        weight = weight * err
        weight /= weight.sum()
    return coef.astype(np.float32)


if __name__ == "__main__":
    for k, c in enumerate(fit()):
        print(f"constexpr float kExp2C{k} = {float(c)!r}f;")
