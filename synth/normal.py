"""Standard normal variates from Philox words by the Box-Muller transform.

Box-Muller (Box and Muller, "A Note on the Generation of Random Normal
Deviates", Ann. Math. Statist. 1958): for u1 in (0, 1] and u2 in [0, 1),
r = sqrt(-2 ln u1) and (r cos 2*pi*u2, r sin 2*pi*u2) are two independent
N(0, 1) deviates.

The logarithm, sine and cosine here are written out from their series using
only IEEE-754 double add, multiply, divide and square root, each correctly
rounded and never fused, evaluated in a fixed order. The device twin in
``synth/csrc/synth_gen.cu`` performs the same operations in the same order, so
both sides produce bit-identical doubles. Accuracy (about 1e-15 relative) is
checked against numpy's libm in the tests; bit-identity with libm is neither
needed nor claimed.

  ln m, m in [1/sqrt2, sqrt2):  ln m = 2 atanh(s), s = (m-1)/(m+1),
                                atanh(s) = sum_k s^(2k+1) / (2k+1)
  sin t, cos t, t in [0, pi/2]: Maclaurin series, Horner form in t^2
"""
import numpy as np

LN2 = 0.6931471805599453          # nearest double to ln 2
HALF_PI = 1.5707963267948966      # nearest double to pi / 2
SQRT2 = 1.4142135623730951        # nearest double to sqrt 2
TWO_M32 = 2.0 ** -32
TWO_M30 = 2.0 ** -30
N_ATANH = 12                      # terms k = 0..11 of the atanh series
N_TRIG = 13                       # terms k = 0..12 of the sin / cos series


def _atanh_coeffs():
    return [1.0 / float(2 * k + 1) for k in range(N_ATANH)]


def _sin_coeffs():
    c = [1.0]
    for k in range(1, N_TRIG):
        c.append(c[-1] / (-float((2 * k) * (2 * k + 1))))
    return c


def _cos_coeffs():
    c = [1.0]
    for k in range(1, N_TRIG):
        c.append(c[-1] / (-float((2 * k - 1) * (2 * k))))
    return c


ATANH_C = _atanh_coeffs()
SIN_C = _sin_coeffs()
COS_C = _cos_coeffs()


def _horner(coeffs, t):
    p = np.full_like(t, coeffs[-1])
    for c in reversed(coeffs[:-1]):
        p = p * t
        p = p + c
    return p


def ln_u1(x):
    """ln((x + 1) * 2^-32) for uint32 x, in float64."""
    n = np.asarray(x, dtype=np.uint64).astype(np.float64) + 1.0   # exact
    m, e = np.frexp(n)                       # n = m 2^e, m in [0.5, 1): exact
    m = m * 2.0                              # [1, 2): exact
    e = e.astype(np.float64) - 1.0
    big = m > SQRT2
    m = np.where(big, m * 0.5, m)            # exact
    e = np.where(big, e + 1.0, e)
    s = (m - 1.0) / (m + 1.0)
    s2 = s * s
    p = _horner(ATANH_C, s2)
    lnm = (2.0 * s) * p
    return (e - 32.0) * LN2 + lnm


def sincos_2pi_u2(x):
    """(sin, cos) of 2*pi*x*2^-32 for uint32 x, in float64."""
    x = np.asarray(x, dtype=np.uint32)
    quad = (x >> np.uint32(30)).astype(np.int64)
    f = (x & np.uint32(0x3FFFFFFF)).astype(np.float64) * TWO_M30    # exact
    th = f * HALF_PI
    t = th * th
    s = th * _horner(SIN_C, t)
    c = _horner(COS_C, t)
    sin_out = np.select([quad == 0, quad == 1, quad == 2], [s, c, -s], -c)
    cos_out = np.select([quad == 0, quad == 1, quad == 2], [c, -s, -c], s)
    return sin_out, cos_out


def box_muller(xa, xb):
    """Two float64 N(0,1) arrays from uint32 word arrays (xa -> u1, xb -> u2)."""
    r = np.sqrt(-2.0 * ln_u1(xa))
    sn, cs = sincos_2pi_u2(xb)
    return r * cs, r * sn
