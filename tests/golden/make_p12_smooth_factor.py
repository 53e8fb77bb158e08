"""Writes p12_smooth_factor_sequences.txt: the fp32 smoothing factor s_j and
its reciprocal for alpha in {0, 1/4, 1/2, 3/4, 1}, worked in exact rational
arithmetic.

The SmoothQuant glossary page (jisaku.com, "Hyper-parameter alpha
(migration strength)") defines s_j = max|X_j|^alpha / max|W_j|^(1-alpha) and
says nothing about how the power is evaluated in floating point.  The
reading used on both sides of the parity check fixes one IEEE fp32 sequence
per alpha (each operation correctly rounded, ties to even):

    alpha = 1     s = a
    alpha = 0     s = 1 / w
    alpha = 1/2   s = sqrt(a) / sqrt(w)
    alpha = 1/4   s = sqrt(sqrt(a)) / (sqrt(w) * sqrt(sqrt(w)))
    alpha = 3/4   s = (sqrt(a) * sqrt(sqrt(a))) / sqrt(sqrt(w))
    inv_s = 1 / s

This script evaluates those sequences with Python's Fraction type: every
intermediate is an exact rational, and each operation is followed by an
explicit round-to-nearest-even onto the fp32 grid (a correctly rounded
square root is found from an integer square root and checked against the
two neighbouring midpoints).  It uses no floating-point arithmetic, no
oracle and no GPU code.

The inputs were picked so that the plausible alternatives -- sqrt(a/w),
sqrt(a) * (1/sqrt(w)), sqrt(sqrt(a/w^3)), (a^3)^(1/4) / w^(1/4), the power
evaluated in double and rounded once, and inv_s from the reciprocal formula
-- each give a different fp32 value; the test checks that too.

Usage: python tests/golden/make_p12_smooth_factor.py  (rewrites the table)
"""
from fractions import Fraction
import math
import os

HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "p12_smooth_factor_sequences.txt")

# (alpha, a, w) with a, w fp32 values written exactly (float.hex)
CASES = [
    (0.25, "0x1.f87132p+2", "0x1.5d28acp-9"),
    (0.25, "0x1.c00022p-5", "0x1.59d43ap-9"),
    (0.25, "0x1.43f07p+3", "0x1.ae094cp-7"),
    (0.5, "0x1.190324p+1", "0x1.da71dcp-3"),
    (0.5, "0x1.4789eap-2", "0x1.19037ep-6"),
    (0.5, "0x1.aa2588p-4", "0x1.8c621ep-7"),
    (0.75, "0x1.0cd642p+2", "0x1.48441cp-6"),
    (0.75, "0x1.290d5ep+4", "0x1.e041d8p-4"),
    (0.75, "0x1.06fb9p-3", "0x1.7ddbcp-5"),
    (1.0, "0x1.190324p+1", "0x1.da71dcp-3"),
    (0.0, "0x1.190324p+1", "0x1.da71dcp-3"),
]


def fl(q: Fraction) -> Fraction:
    """q rounded to the nearest fp32 value, ties to even (normal range)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    assert -126 <= e <= 127, "outside the normal fp32 range"
    ulp = Fraction(2) ** (e - 23)
    n, r = divmod(a, ulp)
    if r > ulp / 2 or (r == ulp / 2 and n % 2 == 1):
        n += 1
    return sign * n * ulp


def _neighbours(r: Fraction):
    """The fp32 values just below and just above the positive fp32 value r."""
    e = r.numerator.bit_length() - r.denominator.bit_length()
    while Fraction(2) ** e > r:
        e -= 1
    while Fraction(2) ** (e + 1) <= r:
        e += 1
    up = Fraction(2) ** (e - 23)
    down = up / 2 if r == Fraction(2) ** e else up
    return r - down, r + up


def fl_sqrt(q: Fraction) -> Fraction:
    """The correctly rounded fp32 square root of q > 0."""
    k = 200
    approx = Fraction(math.isqrt(q.numerator * 4 ** k // q.denominator), 2 ** k)
    r = fl(approx)
    lo, hi = _neighbours(r)
    m_lo, m_hi = (lo + r) / 2, (r + hi) / 2
    # r is the nearest fp32 value iff sqrt(q) lies strictly between the midpoints
    assert m_lo * m_lo < q < m_hi * m_hi, "square root not bracketed"
    return r


def smooth_factor(alpha: float, a: Fraction, w: Fraction) -> Fraction:
    if alpha == 1.0:
        return a
    if alpha == 0.0:
        return fl(1 / w)
    if alpha == 0.5:
        return fl(fl_sqrt(a) / fl_sqrt(w))
    if alpha == 0.25:
        a14 = fl_sqrt(fl_sqrt(a))
        w34 = fl(fl_sqrt(w) * fl_sqrt(fl_sqrt(w)))
        return fl(a14 / w34)
    if alpha == 0.75:
        a34 = fl(fl_sqrt(a) * fl_sqrt(fl_sqrt(a)))
        w14 = fl_sqrt(fl_sqrt(w))
        return fl(a34 / w14)
    raise ValueError(alpha)


def main():
    lines = [
        "# Smoothing factor s = a^alpha / w^(1-alpha) and inv_s = 1/s in fp32, by the",
        "# fixed IEEE sequence of square roots, one product and one division per alpha",
        "# (SmoothQuant glossary page, jisaku.com, \"Hyper-parameter alpha\"; the",
        "# sequence is this build's reading of how the power is evaluated).",
        "# Worked in exact rational arithmetic with explicit round-to-nearest-even by",
        "# tests/golden/make_p12_smooth_factor.py.  Values are float.hex of fp32 numbers.",
        "# Each case: alpha a w s inv_s",
    ]
    for i, (alpha, ah, wh) in enumerate(CASES):
        a, w = Fraction(float.fromhex(ah)), Fraction(float.fromhex(wh))
        assert fl(a) == a and fl(w) == w, "inputs must be fp32 values"
        s = smooth_factor(alpha, a, w)
        inv = fl(1 / s)
        lines.append(f"case{i:02d}: " + " ".join([repr(alpha), ah, wh, float(s).hex(), float(inv).hex()]))
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(OUT)


if __name__ == "__main__":
    main()
