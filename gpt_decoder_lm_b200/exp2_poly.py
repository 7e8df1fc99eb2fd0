"""Coefficients of the polynomial 2^x that the attention kernels evaluate on
the FMA pipe for part of the softmax exponentials (csrc/common.cuh,
exp2_poly2), derived here so that the constants in the CUDA source can be
checked against their derivation (tests/test_exp2_poly.py).

Method (Cody and Waite's argument reduction, 1980; Chebyshev interpolation):
x = n + f with n = round(x) and f in [-1/2, 1/2]; 2^x = 2^n * 2^f, where 2^n
is an exponent-field add and 2^f is the polynomial that interpolates 2^f at
the DEGREE + 1 Chebyshev nodes of [-1/2, 1/2] (near-minimax).  For degree 4
its relative error is below 3.6e-6 over the interval: far below the bf16
rounding (2^-9) of the probabilities it feeds.
"""

import numpy as np

DEGREE = 4


def coefficients(degree: int = DEGREE) -> np.ndarray:
    """Monomial coefficients c_0..c_degree of the Chebyshev interpolant of
    2^f on [-1/2, 1/2] (float64)."""
    k = np.arange(degree + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (degree + 1)))
    vander = np.vander(nodes, degree + 1, increasing=True)
    return np.linalg.solve(vander, 2.0 ** nodes)


def evaluate_f32(x: np.ndarray, degree: int = DEGREE) -> np.ndarray:
    """The device function's arithmetic in float32 (round-to-nearest): the
    reference the CPU test holds the derivation to."""
    c = coefficients(degree).astype(np.float32)
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))   # keeps the exponent field >= 1
    magic = np.float32(12582912.0)                  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)              # round(x) in the low mantissa bits
    n = t.view(np.int32) - magic.view(np.int32)
    f = (x - (t - magic)).astype(np.float32)
    p = np.full_like(f, c[-1])
    for cc in c[-2::-1]:
        # a fused multiply-add: the float32 product is exact in float64
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(cc)).astype(np.float32)
    return (p.view(np.int32) + (n << 23)).view(np.float32)


if __name__ == "__main__":
    for i, v in enumerate(coefficients().astype(np.float32)):
        print(f"c{i} = {float(v)!r}f")
