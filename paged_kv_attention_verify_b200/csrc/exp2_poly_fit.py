"""Derive the polynomial the prefill kernel uses to evaluate part of its exp2 calls on the
FMA pipe (the special-function unit is the prefill softmax's bottleneck on B200).

Method: range reduction 2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2], and a
degree-3 polynomial that interpolates 2^f at the four Chebyshev nodes of [-1/2, 1/2]
(Chebyshev interpolation, which is within a small factor of the minimax polynomial). Run
this file to print the coefficients and the worst relative error on a fine grid; the
kernel's constants (kExp2C0..kExp2C3 in pkva_prefill_body.cuh) are its output, and the CPU test
tests/test_exp2_poly.py re-derives them and checks the error bound.
"""
import numpy as np

DEGREE = 3


def coefficients(degree: int = DEGREE):
    k = np.arange(degree + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (degree + 1)))
    # exact interpolation through the nodes; highest power first
    return np.polyfit(nodes, np.exp2(nodes), degree)


def max_rel_error(c, n=200001):
    f = np.linspace(-0.5, 0.5, n)
    return float(np.max(np.abs(np.polyval(c, f) / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = coefficients()
    for i, v in enumerate(c[::-1]):
        print(f"c{i} = {np.float32(v)!r}  ({v:.17g})")
    print("max relative error on [-1/2, 1/2]:", max_rel_error(c))
