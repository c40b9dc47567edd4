"""Fit of the degree-3 polynomial p(f) ~ 2^f, |f| <= 1/2, used for part of the
attention softmax's exponentials on the FMA pipe (exp2_poly.cuh).

    python patch_diffusion_unet_b200/csrc/exp2_poly_fit.py

Method: the minimax fit in relative error, reached by Lawson's algorithm --
iteratively reweighted least squares, each weight multiplied by the current
absolute relative error and renormalised -- on 256 Chebyshev nodes of [-1/2, 1/2].
With the range reduction 2^x = 2^j * 2^f (j = rint(x)) the relative error of
2^x is that of p on [-1/2, 1/2].  Prints the coefficients (highest power first,
rounded to fp32, the values the kernel holds) and their maximum relative error
on a dense grid.  Written from the mathematics; no library exp2 code is used.
"""
import numpy as np

NODES = 256
ITERATIONS = 200
DEGREE = 3


def fit(nodes=NODES, iterations=ITERATIONS, degree=DEGREE):
    """Coefficients (highest power first, fp64) of the minimax relative-error fit."""
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))
    A = np.vander(f, degree + 1)
    y = 2.0 ** f
    w = np.full(nodes, 1.0 / nodes)
    c = None
    for _ in range(iterations):
        sw = np.sqrt(w) / y                      # relative error: residual divided by 2^f
        c, *_ = np.linalg.lstsq(A * sw[:, None], y * sw, rcond=None)
        e = np.abs(A @ c / y - 1.0)
        w = w * e
        w /= w.sum()
    return c


def max_rel_error(coeffs, samples=200001):
    f = np.linspace(-0.5, 0.5, samples)
    return float(np.max(np.abs(np.polyval(np.asarray(coeffs, np.float64), f) / 2.0 ** f - 1.0)))


def fp32_coefficients():
    return [float(np.float32(v)) for v in fit()]


if __name__ == "__main__":
    c32 = fp32_coefficients()
    print("coefficients (f^3, f^2, f, 1), fp32:", ", ".join(f"{v:.9g}f" for v in c32))
    print(f"max relative error on [-1/2, 1/2]: {max_rel_error(c32):.4e}")
