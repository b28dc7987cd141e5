"""Exact rational model of binary32 round-to-nearest-even and of the two FP
formats of NVFP4, for deriving pinned test values by hand.

Everything here is written from the IEEE-754 binary32 definition (24-bit
significand, exponents -126..127, subnormals down to 2^-149, ties to the even
significand) and from the format definitions of E4M3 (bias 7, 3 mantissa bits,
subnormals m * 2^-9, largest finite 448) and E2M1 (magnitudes 0, 0.5, 1, 1.5,
2, 3, 4, 6; "Four Over Six (4/6)" technical summary, section 문제 제기).  It
shares nothing with the C oracle or the CUDA library: values are Python
Fractions, every rounding is spelled out, and the test files use it only to
derive the expected bits of hand-chosen blocks.
"""
from __future__ import annotations

import math
from fractions import Fraction

INF = float("inf")
_MIN_EXP = -126          # smallest normal exponent
_P = 24                  # significand bits, hidden bit included


def _floor_log2(a: Fraction) -> int:
    """e with 2^e <= a < 2^(e+1), for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def rn32(q):
    """Round a rational to the nearest binary32 value, ties to the even
    significand.  Returns a Fraction, or +-INF on overflow."""
    q = Fraction(q)
    if q == 0:
        return Fraction(0)
    neg = q < 0
    a = -q if neg else q
    e = max(_floor_log2(a), _MIN_EXP)
    ulp = Fraction(2) ** (e - (_P - 1))
    n = a / ulp
    k = n.numerator // n.denominator
    rem = n - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    r = k * ulp
    if r >= Fraction(2) ** 128:
        return -INF if neg else INF
    return -r if neg else r


def is_binary32(q) -> bool:
    return rn32(q) == Fraction(q)


def f32_bits(q) -> int:
    """Bit pattern of a binary32 value given exactly as a Fraction (or INF)."""
    import struct

    if q in (INF, -INF):
        return 0x7F800000 | (0x80000000 if q < 0 else 0)
    assert is_binary32(q), q
    return struct.unpack("<I", struct.pack("<f", float(q)))[0]


def from_bits(b: int) -> Fraction:
    import struct

    return Fraction(struct.unpack("<f", struct.pack("<I", b))[0])


# ------------------------------------------------------------------ E4M3 --

def e4m3_value(code: int) -> Fraction:
    e, m = (code >> 3) & 15, code & 7
    assert not (e == 15 and m == 7), "NaN code"
    v = Fraction(m, 512) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if code & 0x80 else v


_E4M3 = [e4m3_value(c) for c in range(0x7F)]  # 0x00 .. 0x7E, increasing


def e4m3_rne_satfinite(v) -> int:
    """Non-negative value -> nearest finite E4M3 code, ties to the even code,
    anything above 448 -> 448 (0x7E)."""
    v = Fraction(v)
    assert v >= 0
    if v >= _E4M3[-1]:
        return 0x7E
    for c in range(0x7E):
        lo, hi = _E4M3[c], _E4M3[c + 1]
        if v <= hi:
            mid = (lo + hi) / 2
            if v < mid:
                return c
            if v > mid:
                return c + 1
            return c if c % 2 == 0 else c + 1
    raise AssertionError("unreachable")


# ------------------------------------------------------------------ E2M1 --

E2M1_MAGS = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
             Fraction(4), Fraction(6)]


def e2m1_value(code: int) -> Fraction:
    m = E2M1_MAGS[code & 7]
    return -m if code & 8 else m


def e2m1_rne_satfinite(v, negative: bool) -> int:
    """Magnitude |v| -> nearest E2M1 code, ties to the even code, >= 6 -> 6;
    bit 3 carries the sign (`negative`), zero included."""
    a = abs(Fraction(v)) if v not in (INF, -INF) else None
    sign = 8 if negative else 0
    if a is None or a >= 6:
        return sign | 7
    for c in range(7):
        lo, hi = E2M1_MAGS[c], E2M1_MAGS[c + 1]
        if a <= hi:
            mid = (lo + hi) / 2
            if a < mid:
                return sign | c
            if a > mid:
                return sign | (c + 1)
            return sign | (c if c % 2 == 0 else c + 1)
    raise AssertionError("unreachable")


# ---------------------------------------------------- the block step ------

def pairwise16(t):
    """Contiguous pairwise tree ((t0+t1)+(t2+t3))+..., each add rounded."""
    a = list(t)
    while len(a) > 1:
        a = [rn32(a[2 * i] + a[2 * i + 1]) for i in range(len(a) // 2)]
    return a[0]


def sequential16(t):
    """Left-to-right sum (((t0+t1)+t2)+t3)+..., each add rounded."""
    s = t[0]
    for v in t[1:]:
        s = rn32(s + v)
    return s


def candidate(x, alpha, Q, rule, *, quotient="product_first", scaling="reciprocal",
              summation="pairwise"):
    """One scale candidate of one 16-element block, every step one binary32
    rounding.  `x` is 16 binary32 values (Fractions; negative zero given as
    the string "-0"), alpha a binary32 value, Q 6 or 4, rule 'max'|'mae'|'mse'.

    The keyword arguments select the reading of the three steps that the
    pages leave open; the defaults are this library's readings:
      quotient   'product_first': s_raw = fl(b / fl(alpha*Q))
                 'alpha_first':   s_raw = fl(fl(b / alpha) / Q)
      scaling    'reciprocal':    v = fl(x * fl(1/d))
                 'divide':        v = fl(x / d)
      summation  'pairwise' (contiguous tree) or 'sequential' (left to right)
    Returns (codes[16], scale_code, error, trace) with trace holding the
    intermediate values."""
    neg = [xi == "-0" or (xi != "-0" and Fraction(xi) < 0) for xi in x]
    xv = [Fraction(0) if xi == "-0" else Fraction(xi) for xi in x]
    b = max(abs(v) for v in xv)
    if quotient == "product_first":
        aq = rn32(alpha * Q)
        s_raw = rn32(b / aq)
    else:
        aq = None
        s_raw = rn32(rn32(b / alpha) / Q)
    s = e4m3_rne_satfinite(s_raw)
    d = rn32(e4m3_value(s) * alpha)
    r = None
    if scaling == "reciprocal":
        r = Fraction(0) if d == 0 else rn32(1 / d)
        if r in (INF, -INF):
            r = Fraction(0)
        v = [rn32(xi * r) for xi in xv]
    else:
        v = [Fraction(0) if d == 0 else rn32(xi / d) for xi in xv]
    # a product or quotient keeps the sign of x, zero included
    codes = [e2m1_rne_satfinite(vi, ng) for vi, ng in zip(v, neg)]
    e = [rn32(xi - e2m1_value(c) * d) for xi, c in zip(xv, codes)]  # fma: one rounding
    if rule == "max":
        err = max(abs(ei) for ei in e)
    else:
        t = [abs(ei) if rule == "mae" else rn32(ei * ei) for ei in e]
        err = pairwise16(t) if summation == "pairwise" else sequential16(t)
    trace = dict(b=b, aq=aq, s_raw=s_raw, s=s, d=d, r=r, v=v, e=e)
    return codes, s, err, trace


def block(x, alpha, rule, **reading):
    """Four-Over-Six on one block: (codes, scale_code, chose4, E6, E4)."""
    c6, s6, e6, _ = candidate(x, alpha, 6, rule, **reading)
    c4, s4, e4, _ = candidate(x, alpha, 4, rule, **reading)
    pick4 = e4 < e6
    return (c4 if pick4 else c6), (s4 if pick4 else s6), pick4, e6, e4


# ------------------------------------------------------------ RMSNorm --

def sqrt32(q):
    """Correctly rounded binary32 square root of a rational q >= 0 (ties to
    even): the candidate from the float square root, then its neighbours
    checked against q exactly (midpoint squared vs q)."""
    q = Fraction(q)
    assert q >= 0
    if q == 0:
        return Fraction(0)
    guess = rn32(Fraction(math.sqrt(float(q))))
    import struct

    def step(v, d):
        b = struct.unpack("<I", struct.pack("<f", float(v)))[0] + d
        return Fraction(struct.unpack("<f", struct.pack("<I", b))[0])

    v = guess
    for _ in range(4):  # move to the binary32 value whose rounding interval holds sqrt(q)
        lo, hi = (v + step(v, -1)) / 2, (v + step(v, 1)) / 2
        if lo * lo > q:
            v = step(v, -1)
        elif hi * hi < q:
            v = step(v, 1)
        else:
            break
    lo, hi = (v + step(v, -1)) / 2, (v + step(v, 1)) / 2
    assert lo * lo <= q <= hi * hi
    if lo * lo == q or hi * hi == q:  # a tie: the even significand
        other = step(v, -1) if lo * lo == q else step(v, 1)
        bits = struct.unpack("<I", struct.pack("<f", float(v)))[0]
        return v if bits % 2 == 0 else other
    return v


def bf16_rne(q):
    """Nearest bf16 (8-bit significand, binary32's exponent range) of a
    rational, ties to the even significand, overflow to +-INF; returned as a
    Fraction (or +-INF)."""
    q = Fraction(q)
    if q == 0:
        return Fraction(0)
    neg = q < 0
    a = -q if neg else q
    e = max(_floor_log2(a), _MIN_EXP)
    ulp = Fraction(2) ** (e - 7)
    n = a / ulp
    k = n.numerator // n.denominator
    rem = n - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    r = k * ulp
    if r >= Fraction(2) ** 128:
        return -INF if neg else INF
    return -r if neg else r


def pairwise_sum(t):
    """Contiguous pairwise tree over len(t) terms zero-padded to a power of
    two, each add rounded."""
    a = list(t)
    p = 1
    while p < len(a):
        p *= 2
    a += [Fraction(0)] * (p - len(a))
    while len(a) > 1:
        a = [rn32(a[2 * i] + a[2 * i + 1]) for i in range(len(a) // 2)]
    return a[0]


def rmsnorm_row(x, gamma, eps, *, summation="pairwise", mean="divide", rsqrt="sqrt_then_divide",
                order="x_r_then_gamma"):
    """One row of RMSNorm with every step rounded to binary32, y rounded to
    bf16.  x, gamma: lists of bf16 values as Fractions; eps a binary32 value.
    The keywords select the reading of the steps the pages leave open; the
    defaults are this library's:
      summation  'pairwise' (contiguous tree) | 'sequential'
      mean       'divide': fl(s / K)          | 'reciprocal': fl(s * fl(1/K))
      rsqrt      'sqrt_then_divide': fl(1 / fl(sqrt(d)))
                 | 'rsqrt': the correctly rounded 1/sqrt(d)
      order      'x_r_then_gamma': fl(fl(x*r)*g) | 'r_gamma_first': fl(x*fl(r*g))"""
    r = rms_scale(x, eps, summation=summation, mean=mean, rsqrt=rsqrt)
    return [rms_out(v, r, g, order=order) for v, g in zip(x, gamma)]


def rms_scale(x, eps, *, summation="pairwise", mean="divide", rsqrt="sqrt_then_divide"):
    """The row's factor r = 1 / sqrt(mean(x^2) + eps) under the readings of
    rmsnorm_row."""
    K = len(x)
    t = [rn32(v * v) for v in x]
    s = pairwise_sum(t) if summation == "pairwise" else _seq(t)
    ms = rn32(s / K) if mean == "divide" else rn32(s * rn32(Fraction(1, K)))
    d = rn32(ms + eps)
    return rn32(1 / sqrt32(d)) if rsqrt == "sqrt_then_divide" else _rsqrt32(d)


def rms_out(v, r, g, *, order="x_r_then_gamma"):
    """One output element bf16((v * r) * g) under the product-order reading."""
    if order == "x_r_then_gamma":
        return bf16_rne(rn32(rn32(v * r) * g))
    return bf16_rne(rn32(v * rn32(r * g)))


def _seq(t):
    s = t[0]
    for v in t[1:]:
        s = rn32(s + v)
    return s


def _rsqrt32(d):
    """Correctly rounded binary32 1/sqrt(d), d > 0: the binary32 value v whose
    rounding interval holds 1/sqrt(d), i.e. lo <= 1/sqrt(d) <= hi, checked as
    lo^2 * d <= 1 <= hi^2 * d."""
    import struct

    def step(v, k):
        b = struct.unpack("<I", struct.pack("<f", float(v)))[0] + k
        return Fraction(struct.unpack("<f", struct.pack("<I", b))[0])

    v = rn32(Fraction(1 / math.sqrt(float(d))))
    for _ in range(4):
        lo, hi = (v + step(v, -1)) / 2, (v + step(v, 1)) / 2
        if lo * lo * d > 1:
            v = step(v, -1)
        elif hi * hi * d < 1:
            v = step(v, 1)
        else:
            break
    lo, hi = (v + step(v, -1)) / 2, (v + step(v, 1)) / 2
    assert lo * lo * d <= 1 <= hi * hi * d
    return v


def float_hex(q) -> str:
    """binary32 value as a C99 hex float (exact)."""
    return float(q).hex() if q not in (INF, -INF) else ("inf" if q > 0 else "-inf")


def parse_hex(s: str):
    s = s.strip()
    if s == "-0":
        return "-0"
    return Fraction(float.fromhex(s))


__all__ = [n for n in dir() if not n.startswith("_") and n != "math"]
_ = math
