"""Derive the polynomial constants used by sscan_tiled.cu's phase P (run by hand;
the kernel carries the printed values).

log1p(v) for v in [0, 1] is evaluated as v * p(v), with p the degree-9 Chebyshev
interpolant of log1p(v)/v on [0, 1] (numpy's Chebyshev.interpolate at the
Chebyshev points, then converted to monomial coefficients for Horner's rule).
Its error is 5e-9 in exact arithmetic and below 2e-7 relative once evaluated in
fp32.  The reciprocal seed for 1/d, d in [1, 2], is the degree-1 Chebyshev
interpolant of 1/d (relative error <= 1/17); three Newton steps y <- y + y(1 - d y)
bring it to fp32 rounding.
"""
import numpy as np
from numpy.polynomial import chebyshev as Ch
from numpy.polynomial import polynomial as P


def log1p_over_v(v):
    v = np.asarray(v, dtype=np.float64)
    safe = np.where(v == 0, 1.0, v)
    return np.where(v == 0, 1.0, np.log1p(safe) / safe)


def main():
    c = Ch.Chebyshev.interpolate(log1p_over_v, 9, domain=[0, 1]).convert(kind=P.Polynomial).coef
    print("log1p(v)/v, v^0 .. v^9:")
    for k, x in enumerate(c):
        print(f"  c{k} = {float(np.float32(x)):.9g}f   ({float(x)!r})")
    s = Ch.Chebyshev.interpolate(lambda d: 1.0 / d, 1, domain=[1, 2]).convert(kind=P.Polynomial).coef
    print(f"1/d seed: {float(np.float32(s[0])):.9g}f + {float(np.float32(s[1])):.9g}f * d")
    v = np.linspace(0, 1, 100001)
    print("max rel err of v*p(v):", np.max(np.abs(P.polyval(v, c) * v - np.log1p(v)) / np.maximum(np.log1p(v), 1e-300)))


if __name__ == "__main__":
    main()
