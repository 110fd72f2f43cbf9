"""Exact rational arithmetic for pinning the oracle: IEEE round-to-nearest-even onto a
binary grid, the E2M1 / E4M3 element grids as fractions, and the search for inputs whose
static E4M3 code is decided by less than a binary32 rounding.  Nothing here computes in
floating point; every value is a fractions.Fraction."""
from __future__ import annotations

import struct
from fractions import Fraction

HALF = Fraction(1, 2)


def floor_log2(a: Fraction) -> int:
    """floor(log2 a) for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    return e - 1 if Fraction(2) ** e > a else e


def rn_binary(v: Fraction, p: int, emin: int, emax: int | None = None):
    """v rounded to nearest, ties to even, onto the binary format with p significant bits
    and minimum normal exponent emin (subnormals below 2^emin).  With emax given, results
    at or above 2^(emax + 1) become +-inf (float)."""
    if v == 0:
        return Fraction(0)
    a = abs(v)
    e = max(floor_log2(a), emin)     # a in [2^e, 2^(e+1)), or the subnormal range
    q = Fraction(2) ** (e - p + 1)   # grid spacing
    n = a / q
    f = n.numerator // n.denominator
    rem = n - f
    if rem > HALF or (rem == HALF and f % 2 == 1):
        f += 1
    r = f * q
    if emax is not None and r >= Fraction(2) ** (emax + 1):
        return float("inf") if v > 0 else float("-inf")
    return r if v > 0 else -r


def rn32(v: Fraction):
    """Nearest binary32 value (as a Fraction, or +-inf)."""
    return rn_binary(v, 24, -126, 127)


def f32_fraction(x: float) -> Fraction:
    """The exact value of a binary32 number given as a Python float."""
    return Fraction(struct.unpack("<f", struct.pack("<f", x))[0])


def bf16_fraction(bits: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0])


def bf16_bits(v: Fraction) -> int:
    """bf16 bits of v, which must be exactly representable in bf16."""
    f = float(v)
    u = struct.unpack("<I", struct.pack("<f", f))[0]
    assert u & 0xFFFF == 0 and Fraction(f) == v, v
    return u >> 16


def f32_bits(v: Fraction) -> int:
    f = float(v)
    assert Fraction(f) == v
    return struct.unpack("<I", struct.pack("<f", f))[0]


def _e4m3_mag(code: int) -> Fraction:
    e, m = code >> 3, code & 7
    if e == 0:
        return Fraction(m, 8) * Fraction(2) ** -6
    return (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)


E2M1_GRID = [Fraction(v) for v in (0, HALF, 1, Fraction(3, 2), 2, 3, 4, 6)]
E4M3_GRID = [_e4m3_mag(c) for c in range(0x7F)]  # codes 0..126
GRIDS = {0: (E2M1_GRID, 3), 1: (E4M3_GRID, 7)}   # format -> (magnitudes by code, sign bit)


def nearest_code(v: Fraction, fmt: int, negative: bool | None = None) -> int:
    """Element code of v rounded to nearest on the grid, ties to the even code, values
    past the largest magnitude saturating; the sign bit is set for negative v (and for a
    negative zero when `negative` says so)."""
    grid, sbit = GRIDS[fmt]
    a = abs(v)
    if a >= grid[-1]:
        code = len(grid) - 1
    else:
        lo = max(i for i, g in enumerate(grid) if g <= a)
        hi = lo + 1
        dl, dh = a - grid[lo], grid[hi] - a
        code = lo if (dl < dh or (dl == dh and lo % 2 == 0)) else hi
    neg = v < 0 if negative is None else negative
    return code | (int(neg) << sbit)


def e4m3_midpoints_in_binade():
    """The E4M3 decision boundaries in [1, 2): the midpoints (17 + 2j) / 16."""
    return [Fraction(17 + 2 * j, 16) for j in range(8)]


def static_near_ties():
    """Pairs (s, x) -- s a binary32 scale, x a bf16 value in [1, 2) -- for which the
    exact quotient x / s and a binary32 evaluation of it take different E4M3 codes: the
    correctly rounded binary32 quotient, or the binary32 product x * fl32(1/s), lies on or
    across an E4M3 midpoint from x / s.  Found by exhaustive search over the bf16 values
    x in [1, 2), the midpoints m in [1, 2) and the binary32 scales next to x / m."""
    out = []
    for m in e4m3_midpoints_in_binade():
        for X in range(128, 256):
            x = Fraction(X, 128)
            s0 = rn32(x / m)
            ulp = Fraction(2) ** (floor_log2(s0) - 23)
            for s in (s0 - ulp, s0, s0 + ulp):
                q = x / s
                want = nearest_code(q, 1)
                quo = rn32(q)
                prod = rn32(x * rn32(1 / s))
                if nearest_code(quo, 1) != want or nearest_code(prod, 1) != want:
                    out.append((s, x))
    return out


def hadamard_sign(j: int, k: int) -> int:
    """Entry (j, k) of the Sylvester Hadamard matrix: (-1)^popcount(j & k)."""
    return -1 if bin(j & k).count("1") % 2 else 1


def transform_exact(x_bits, B: int, mul=None):
    """S = (x * mul) . blockdiag(H_B) for one row of bf16 bits, as exact fractions (the
    transformed values are S / sqrt(B))."""
    K = len(x_bits)
    a = [bf16_fraction(int(b)) * (1 if mul is None else f32_fraction(float(mul[k]))) for k, b in enumerate(x_bits)]
    S = []
    for b0 in range(0, K, B):
        for j in range(B):
            S.append(sum(hadamard_sign(j, k) * a[b0 + k] for k in range(B) if a[b0 + k] != 0))
    return S


def scale_code_sqrt(S_block, B: int, emax: int) -> int:
    """E8M0 scale code of a block whose values are S_i / sqrt(B): floor(log2 max|t|) + 127
    - emax, clamped at 0, decided exactly (floor(log2 sqrt(v)) = floor(floor(log2 v) / 2)
    for v = max S_i^2 / B)."""
    m = max(abs(v) for v in S_block)
    if m == 0:
        return 0
    e = floor_log2(m * m / B) // 2
    return max(0, e + 127 - emax)


def nearest_code_sqrt(S: Fraction, B: int, X: Fraction, fmt: int) -> int:
    """Code of t / X on the element grid for t = S / sqrt(B), decided exactly by comparing
    squares: |t / X| >= g  <=>  S^2 >= g^2 X^2 B.  For B an odd power of two sqrt(B) is
    irrational, so t / X never equals a midpoint unless S = 0 (+0 here)."""
    grid, sbit = GRIDS[fmt]
    s2 = S * S
    w = X * X * B
    if s2 >= grid[-1] ** 2 * w:
        code = len(grid) - 1
    else:
        lo = max(i for i, g in enumerate(grid) if g * g * w <= s2)
        mid = (grid[lo] + grid[lo + 1]) / 2
        code = lo + 1 if s2 > mid * mid * w else lo
    return code | (int(S < 0) << sbit)
