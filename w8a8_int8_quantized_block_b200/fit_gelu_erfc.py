"""Coefficients of the GELU epilogue's erfc (gemm_core.cuh, gelu_pair).

erfc(x) for x >= 0 is written as t * exp(-x^2 + g(t)) with t = 1 / (1 + x/2),
the form of the classic Chebyshev-fitted complementary error function
(Numerical Recipes, "erfcc").  g(t) = log(erfcx(x) / t) is smooth on
t in (0, 1]; it is interpolated here at Chebyshev nodes by a polynomial of
degree 7 in t, and the coefficients are scaled by log2(e) so that the kernel
evaluates 2^(log2(e) g(t) - log2(e) x^2).  The form keeps the relative
accuracy of erfc in the tail, where GELU(y) = y Phi(y) of a negative y is
0.5 y erfc(|y| / sqrt 2).

Run: python -m w8a8_int8_quantized_block_b200.fit_gelu_erfc  (prints the
coefficients, highest degree first, and the maximum relative error of GELU
evaluated as the kernel does, in float32, against float64)."""
import numpy as np
from scipy.special import erfc, erfcx

DEG = 7


def fit(deg=DEG):
    n = 4000
    t = 0.5 * (1 - np.cos(np.pi * (np.arange(n) + 0.5) / n))
    x = 2.0 * (1.0 / t - 1.0)
    g = np.log(erfcx(x) / t)
    c = np.polynomial.chebyshev.chebfit(2 * t - 1, g, deg)
    p = np.polynomial.Polynomial(np.polynomial.chebyshev.cheb2poly(c))(np.polynomial.Polynomial([-1.0, 2.0]))
    return (p.coef * np.log2(np.e)).astype(np.float32)  # t^0 .. t^deg, times log2(e)


def gelu_f32(y, c):
    """GELU as the kernel computes it, in float32 (exact division and exp2
    stand in for the approximate reciprocal and 2^x)."""
    y = y.astype(np.float32)
    ay = np.abs(y)
    t = np.float32(1.0) / (ay * np.float32(0.5 / np.sqrt(2.0)) + np.float32(1.0))
    p = np.full_like(t, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = p * t + c[k]
    arg = (ay * np.float32(-0.5 * np.log2(np.e))) * ay + p
    e = t * np.exp2(arg).astype(np.float32)
    h = np.float32(0.5) * y * e
    return np.where(y >= 0, y - h, h)


if __name__ == "__main__":
    c = fit()
    print("coefficients t^%d .. t^0:" % DEG, ", ".join("%.9ef" % v for v in c[::-1]))
    y = np.concatenate([np.linspace(-30, 30, 600001), -np.logspace(-8, 1.5, 20001), np.logspace(-8, 1.5, 20001)])
    ref = 0.5 * y * erfc(-y / np.sqrt(2.0))
    got = gelu_f32(y, c).astype(np.float64)
    ok = np.abs(ref) > 1e-30
    print("max relative error of GELU on [-30, 30]: %.3g" % (np.abs(got[ok] - ref[ok]) / np.abs(ref[ok])).max())
