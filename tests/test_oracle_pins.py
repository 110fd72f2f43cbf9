"""Pins of the CPU oracle against things other than itself.

The MX format is the one the blog "Quark Mixed-Precision Quantization for Wan2.2
Video Generation on AMD Instinct GPUs" uses (section "Quantization formats"): OCP
MXFP4 (E2M1 elements) and FP8 E4M3 elements, 32-element blocks, one E8M0 scale per
block, RTN.  The pins below use independent routes to the same answers:

* element rounding: exhaustive over all bf16 bit patterns against a brute-force
  nearest-value search over the enumerated grids (ties to the even code);
* element grids: literal values from the format tables;
* scale: closed form max(0, j + 127 - emax) for amax in [2^j, 2^(j+1));
* hand-worked blocks: tests/golden/hand_blocks.json;
* invariants: idempotence, power-of-two equivariance, sign symmetry, permutation;
* the linear layer: exact rational brute force on tiny matrices, and the
  lossless case where numpy's fp64 matmul is the answer.
"""
import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import _exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FMT = {"e2m1": oracle.E2M1, "e4m3": oracle.E4M3}


# --- independent descriptions of the element grids ---------------------------------

# E2M1 magnitudes by code 0..7, as listed in the OCP MX element-format table.
E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_mag(code):
    """E4M3 magnitude from its bit fields: exponent bias 7, 3 mantissa bits,
    subnormals m/8 * 2^-6; code 0x7F is NaN and not part of the grid."""
    e, m = code >> 3, code & 7
    if e == 0:
        return m / 8.0 * 2.0 ** -6
    return (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_MAG = [e4m3_mag(c) for c in range(0x7F)]  # codes 0..126 (finite, non-negative)
GRID = {oracle.E2M1: (E2M1_MAG, 3), oracle.E4M3: (E4M3_MAG, 7)}  # (magnitudes, sign bit)


def brute_round(y, fmt):
    """Nearest grid value by exhaustive search; ties to the even code; values past the
    largest magnitude saturate; the sign bit follows the sign of y (even for 0)."""
    mags, sbit = GRID[fmt]
    a = abs(y)
    best = None
    for code, g in enumerate(mags):
        d = abs(a - g)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    code = best[1]
    if a > mags[-1]:
        code = len(mags) - 1
    neg = math.copysign(1.0, y) < 0
    return code | (int(neg) << sbit)


def all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    keep = np.isfinite(f)
    return bits[keep].astype(np.uint16), f[keep].astype(np.float64)


# --- element grids -----------------------------------------------------------------------

def test_e2m1_decode_table():
    for c in range(16):
        want = E2M1_MAG[c & 7] * (-1.0 if c & 8 else 1.0)
        got = oracle.decode_elem(c, oracle.E2M1)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), c


def test_e4m3_decode_table():
    for c in range(256):
        got = oracle.decode_elem(c, oracle.E4M3)
        if c & 0x7F == 0x7F:
            assert math.isnan(got)
            continue
        want = e4m3_mag(c & 0x7F) * (-1.0 if c & 0x80 else 1.0)
        assert got == want, hex(c)
    # a few literal anchors of the format
    assert oracle.decode_elem(0x7E, oracle.E4M3) == 448.0
    assert oracle.decode_elem(0x01, oracle.E4M3) == 2.0 ** -9
    assert oracle.decode_elem(0x08, oracle.E4M3) == 2.0 ** -6
    assert oracle.decode_elem(0x38, oracle.E4M3) == 1.0


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_element_rounding_exhaustive_bf16(fmt):
    """Every finite bf16 value, and every finite bf16 value times 2^-k for small k
    (to sweep the ties and subnormals of the target grid densely), rounds exactly as
    a brute-force nearest search over the grid."""
    _, vals = all_finite_bf16()
    mags = np.array(GRID[fmt][0])
    sbit = GRID[fmt][1]
    for shift in (0, 3, 7):
        ys = vals * 2.0 ** -shift
        a = np.abs(ys)
        d = np.abs(a[:, None] - mags[None, :])
        dmin = d.min(axis=1, keepdims=True)
        ties = d == dmin
        # prefer the even code among the nearest ones
        even = ties & (np.arange(len(mags))[None, :] % 2 == 0)
        code = np.where(even.any(axis=1), even.argmax(axis=1), ties.argmax(axis=1))
        code = np.where(a > mags[-1], len(mags) - 1, code)
        code = code | (np.signbit(ys).astype(np.int64) << sbit)
        got = np.array([oracle.encode_elem(y, fmt) for y in ys])
        bad = np.nonzero(got != code)[0]
        assert bad.size == 0, [(ys[i], got[i], code[i]) for i in bad[:5]]


def test_brute_round_agrees_with_vectorised_search():
    # the two test-side searches must agree with each other on a handful of values
    for fmt in (oracle.E2M1, oracle.E4M3):
        for y in (0.25, 0.75, -1.25, 5.0, 7.0, 1e-30, -0.0, 2.0 ** -10, 464.0, 500.0):
            assert brute_round(y, fmt) == oracle.encode_elem(y, fmt)


# --- the shared scale ---------------------------------------------------------------------

@pytest.mark.parametrize("fmt,emax", [(oracle.E2M1, 2), (oracle.E4M3, 8)])
def test_scale_code_closed_form(fmt, emax):
    for j in range(-133, 128):
        for mant in (1.0, 1.5, 2.0 - 2.0 ** -7):
            amax = mant * 2.0 ** j
            assert oracle.scale_code(amax, fmt) == max(0, j + 127 - emax), (j, mant)
    assert oracle.scale_code(0.0, fmt) == 0
    assert oracle.scale_code(1.0, fmt, nonfinite=True) == 255


# --- hand-worked blocks -------------------------------------------------------------------

def _expand(runs):
    out = []
    for v, n in runs:
        out += [float.fromhex(v) if isinstance(v, str) else v] * n
    return out


def _bf16_bits(vals):
    return np.array([struct.unpack("<I", struct.pack("<f", v))[0] >> 16 for v in vals],
                    dtype=np.uint16)


def load_hand_blocks():
    with open(os.path.join(GOLDEN, "hand_blocks.json")) as f:
        return json.load(f)["blocks"]


@pytest.mark.parametrize("blk", load_hand_blocks(), ids=lambda b: b["name"])
def test_hand_worked_block(blk):
    fmt = FMT[blk["fmt"]]
    x = _expand(blk["x"])
    assert len(x) == 32
    bits = _bf16_bits(x)
    assert all(oracle.bf16_to_float(int(b)) == v for b, v in zip(bits, x))
    codes, sf = oracle.quantize(bits[None, :], fmt)
    assert int(sf[0, 0]) == blk["sf"]
    want = _expand(blk["codes"])
    if fmt == oracle.E4M3:
        got = list(codes[0])
    else:
        got = []
        for b in codes[0]:
            got += [int(b) & 0xF, int(b) >> 4]
    assert got == want
    if "packed_first_bytes" in blk:
        n = len(blk["packed_first_bytes"])
        assert list(codes[0, :n]) == blk["packed_first_bytes"]


# --- invariants ---------------------------------------------------------------------------

def _random_blocks(rng, nblk, scale_spread=6):
    x = rng.standard_normal((nblk, 32)) * 2.0 ** rng.integers(-scale_spread, scale_spread, (nblk, 1))
    x[rng.random((nblk, 32)) < 0.05] *= 40.0
    return _bf16_bits(x.astype(np.float32).ravel()).reshape(nblk, 32)


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_idempotence(fmt):
    rng = np.random.default_rng(1)
    bits = _random_blocks(rng, 2000)
    codes, sf = oracle.quantize(bits, fmt)
    deq = oracle.dequantize(codes, sf, 32, fmt)
    deq_bits = _bf16_bits(deq.astype(np.float32).ravel()).reshape(deq.shape)
    assert np.array_equal(deq, deq_bits_to_f64(deq_bits))  # exact in bf16
    codes2, sf2 = oracle.quantize(deq_bits, fmt)
    keep = sf[:, 0] > 0
    assert keep.all()
    assert np.array_equal(sf2, sf)
    # a zero element may flip between +0 and -0 only if its input was +-0; none here
    assert np.array_equal(codes2, codes)


def deq_bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_power_of_two_equivariance(fmt):
    rng = np.random.default_rng(2)
    bits = _random_blocks(rng, 500, scale_spread=3)
    x = deq_bits_to_f64(bits)
    codes, sf = oracle.quantize(bits, fmt)
    for j in (-5, -1, 1, 7):
        codes_j, sf_j = oracle.quantize(_bf16_bits((x * 2.0 ** j).astype(np.float32).ravel())
                                        .reshape(bits.shape), fmt)
        assert np.array_equal(codes_j, codes)
        assert np.array_equal(sf_j.astype(int), sf.astype(int) + j)


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_sign_symmetry(fmt):
    rng = np.random.default_rng(3)
    bits = _random_blocks(rng, 500)
    codes, sf = oracle.quantize(bits, fmt)
    codes_n, sf_n = oracle.quantize(bits ^ np.uint16(0x8000), fmt)
    assert np.array_equal(sf_n, sf)
    flip = 0x88 if fmt == oracle.E2M1 else 0x80
    assert np.array_equal(codes_n, codes ^ np.uint8(flip))


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_permutation_within_block(fmt):
    rng = np.random.default_rng(4)
    bits = _random_blocks(rng, 200)
    codes, sf = oracle.quantize(bits, fmt)
    perm = rng.permutation(32)
    codes_p, sf_p = oracle.quantize(bits[:, perm], fmt)
    assert np.array_equal(sf_p, sf)
    unpack = lambda c: (np.stack([c & 0xF, c >> 4], -1).reshape(c.shape[0], -1)
                        if fmt == oracle.E2M1 else c)
    assert np.array_equal(unpack(codes_p), unpack(codes)[:, perm])


def test_nonfinite_block_convention():
    x = [1.0] * 32
    x[5] = float("inf")
    codes, sf = oracle.quantize(_bf16_bits(x)[None, :], oracle.E2M1)
    assert sf[0, 0] == 255 and not codes.any()
    assert math.isnan(oracle.dequantize(codes, sf, 32, oracle.E2M1)[0, 0])


# --- tiled scale layout -----------------------------------------------------------------------

def test_sf_tiled_layout_hand_offsets():
    # K = 256 -> 8 k-blocks -> 2 atoms along k per 128-row tile
    K = 256
    assert oracle.sf_tiled_offset(0, 0, K) == 0
    assert oracle.sf_tiled_offset(0, 3, K) == 3
    assert oracle.sf_tiled_offset(1, 0, K) == 16
    assert oracle.sf_tiled_offset(32, 0, K) == 4
    assert oracle.sf_tiled_offset(97, 2, K) == 16 + 12 + 2
    assert oracle.sf_tiled_offset(0, 4, K) == 512
    assert oracle.sf_tiled_offset(128, 0, K) == 1024
    assert oracle.sf_tiled_offset(130, 5, K) == 1024 + 512 + 2 * 16 + 1


@pytest.mark.parametrize("rows,K", [(1, 32), (127, 96), (129, 160), (300, 1024)])
def test_sf_tiled_layout_is_injective_and_padded(rows, K):
    KB = K // 32
    rng = np.random.default_rng(rows)
    sf = rng.integers(1, 255, (rows, KB), dtype=np.uint8)
    t = oracle.sf_to_tiled(sf, K)
    assert t.size == ((rows + 127) // 128) * 128 * ((KB + 3) // 4) * 4
    offs = {oracle.sf_tiled_offset(r, kb, K) for r in range(rows) for kb in range(KB)}
    assert len(offs) == rows * KB
    assert np.count_nonzero(t) == rows * KB  # padding bytes are zero
    for r in (0, rows - 1):
        for kb in (0, KB - 1):
            assert t[oracle.sf_tiled_offset(r, kb, K)] == sf[r, kb]


# --- the linear layer -------------------------------------------------------------------------

def _exact_value(code, sfc, fmt):
    mags, sbit = GRID[fmt]
    mag = Fraction(mags[code & ((1 << sbit) - 1)])
    v = mag * Fraction(2) ** (sfc - 127)
    return -v if code >> sbit & 1 else v


def _codes_list(codes, K, fmt):
    if fmt == oracle.E4M3:
        return [int(c) for c in codes[:K]]
    out = []
    for b in codes:
        out += [int(b) & 0xF, int(b) >> 4]
    return out


@pytest.mark.parametrize("M,N,K,fmt", [(3, 4, 32, oracle.E2M1), (4, 2, 64, oracle.E2M1),
                                       (2, 3, 64, oracle.E4M3), (1, 1, 32, oracle.E4M3)])
def test_linear_brute_force_exact(M, N, K, fmt):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    x = _bf16_bits((rng.standard_normal((M, K)) * 3).astype(np.float32).ravel()).reshape(M, K)
    w = _bf16_bits((rng.standard_normal((N, K)) * 0.05).astype(np.float32).ravel()).reshape(N, K)
    b = _bf16_bits(rng.standard_normal(N).astype(np.float32))
    xc, xs = oracle.quantize(x, fmt)
    wc, ws = oracle.quantize(w, oracle.E2M1)
    y = oracle.linear(xc, xs, fmt, K, wc, ws, b)
    for m in range(M):
        xa = _codes_list(xc[m], K, fmt)
        for n in range(N):
            wa = _codes_list(wc[n], K, oracle.E2M1)
            acc = Fraction(0)
            for k in range(K):
                acc += (_exact_value(xa[k], int(xs[m, k // 32]), fmt) *
                        _exact_value(wa[k], int(ws[n, k // 32]), oracle.E2M1))
            acc += Fraction(oracle.bf16_to_float(int(b[n])))
            assert abs(float(acc) - y[m, n]) <= 1e-12 * max(1.0, abs(float(acc))), (m, n)


def _mx_representable(rng, rows, K, fmt):
    """Random bf16 matrices that are exactly MX-representable: random element codes
    with one block element forced to the largest magnitude, and random scales."""
    mags, sbit = GRID[fmt]
    KB = K // 32
    codes = rng.integers(0, len(mags), (rows, K))
    codes[:, ::32] = len(mags) - 1
    signs = rng.integers(0, 2, (rows, K))
    sfc = rng.integers(110, 135, (rows, KB))
    vals = np.array(mags)[codes] * np.where(signs, -1.0, 1.0) * 2.0 ** (np.repeat(sfc, 32, 1) - 127)
    return _bf16_bits(vals.astype(np.float32).ravel()).reshape(rows, K), vals, sfc


@pytest.mark.parametrize("fmt", [oracle.E2M1, oracle.E4M3])
def test_linear_lossless_case_matches_numpy(fmt):
    rng = np.random.default_rng(11)
    M, N, K = 37, 29, 256
    xb, xv, xsf = _mx_representable(rng, M, K, fmt)
    wb, wv, wsf = _mx_representable(rng, N, K, oracle.E2M1)
    xc, xs = oracle.quantize(xb, fmt)
    wc, ws = oracle.quantize(wb, oracle.E2M1)
    assert np.array_equal(xs.astype(int), xsf) and np.array_equal(ws.astype(int), wsf)
    assert np.array_equal(oracle.dequantize(xc, xs, K, fmt), xv)
    y = oracle.linear(xc, xs, fmt, K, wc, ws)
    ref = xv @ wv.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-300)
    # rows subset and multi-threaded split give the same numbers
    rows = np.array([36, 0, 17])
    y2 = oracle.linear_rows(xc, xs, fmt, rows, K, wc, ws, nthreads=3)
    assert np.array_equal(y2, y[rows])


# --- the FFN hidden activation: bf16 rounding and GELU --------------------------------------
#
# Pins for the two elementwise steps between a FFN's linears (y -> bf16 -> GELU -> bf16):
# IEEE round-to-nearest-even onto the bf16 grid, and GELU(x) = x * Phi(x) in its erf form.

def _bf16_value(bits):
    return float(np.array([int(bits) << 16], dtype=np.uint32).view(np.float32)[0])


def test_bf16_round_fixed_points():
    """Every finite bf16 value (both zeros, subnormals, the largest) rounds to itself."""
    bits, vals = all_finite_bf16()
    got = oracle.round_bf16(vals)
    assert np.array_equal(got, bits)


def test_bf16_round_midpoints_go_to_even():
    """The exact midpoint of two neighbouring bf16 values rounds to the one with an even
    last fraction bit; a hair off the midpoint it rounds to the nearer one."""
    lo = np.arange(0x0000, 0x7F7F, 97, dtype=np.uint32)  # positive finite, neighbour lo+1 finite
    for s in (0, 0x8000):
        for b in lo:
            a, c = _bf16_value(b | s), _bf16_value((b + 1) | s)
            mid = (a + c) / 2.0  # exact in double
            even = b if b % 2 == 0 else b + 1
            assert oracle.double_to_bf16(mid) == (even | s), hex(b | s)
            assert oracle.double_to_bf16(math.nextafter(mid, a)) == (b | s)
            assert oracle.double_to_bf16(math.nextafter(mid, c)) == ((b + 1) | s)


def test_bf16_round_matches_integer_rounding_of_binary32():
    """For values that are binary32 numbers, rounding to bf16 is the rounding of the
    low 16 bits of the binary32 pattern to even: an integer formula independent of the
    oracle's arithmetic."""
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    keep = np.isfinite(f) & (np.abs(f) <= np.float32(3.3895313892515355e38))  # no overflow
    u, f = u[keep], f[keep]
    want = ((u.astype(np.uint64) + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    got = oracle.round_bf16(f.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_round_nearest_on_random_doubles():
    """Doubles with more precision than binary32: the result is the nearer of the two
    bf16 neighbours that bracket the value."""
    rng = np.random.default_rng(12)
    vals = rng.standard_normal(5000) * np.exp2(rng.integers(-140, 120, size=5000))
    for v in vals:
        r = oracle.double_to_bf16(v)
        rv = _bf16_value(r)
        for nb in (r - 1, r + 1):
            if (nb & 0x7FFF) < 0x7F80 and (nb & 0x8000) == (r & 0x8000):
                assert abs(v - rv) <= abs(v - _bf16_value(nb)), (v, hex(r))


def test_bf16_round_overflow_and_nan():
    top = _bf16_value(0x7F7F)                        # largest finite bf16, odd fraction
    mid = (top + 2.0 ** 128) / 2.0                   # its midpoint with 2^128
    assert oracle.double_to_bf16(mid) == 0x7F80      # tie goes to even: past the top -> Inf
    assert oracle.double_to_bf16(math.nextafter(mid, 0.0)) == 0x7F7F
    assert oracle.double_to_bf16(-mid) == 0xFF80
    assert oracle.double_to_bf16(float("inf")) == 0x7F80
    assert oracle.double_to_bf16(float("nan")) & 0x7FC0 == 0x7FC0
    assert oracle.double_to_bf16(2.0 ** -134) == 0x0000  # half the smallest subnormal: tie to even 0
    assert oracle.double_to_bf16(3 * 2.0 ** -134) == 0x0002  # 1.5 x smallest: tie to even (2)


def test_gelu_is_x_times_normal_cdf():
    """GELU(x) = x * Phi(x), Phi the standard normal CDF (scipy's ndtr)."""
    from scipy.special import ndtr
    xs = np.concatenate([np.linspace(-9.0, 9.0, 3601), [1e-300, -1e-300, 37.5, -5.5]])
    for x in xs:
        want = x * ndtr(x)
        got = oracle.gelu(x)
        assert abs(got - want) <= 2e-14 * max(abs(want), 1e-300) + 1e-300, (x, got, want)


def test_gelu_reflection_and_limits():
    """GELU(x) - GELU(-x) = x; GELU(0) = 0; GELU(x) = x once Phi(x) rounds to 1."""
    for x in np.linspace(-6.0, 6.0, 1201):
        assert abs((oracle.gelu(x) - oracle.gelu(-x)) - x) <= 1e-15 * max(1.0, abs(x)), x
    assert oracle.gelu(0.0) == 0.0
    assert oracle.gelu(10.0) == 10.0


def test_gelu_bf16_hand_values():
    """Worked by hand: GELU(1) = 0.84134..., bf16 spacing 2^-8 there, nearest 0.83984375
    (0x3F57); GELU(-1) = -0.15865..., spacing 2^-10, nearest -0.158203125 (0xBE22);
    GELU(2) = 1.95449..., spacing 2^-7, nearest 1.953125 (0x3FFA)."""
    y = np.array([0x3F80, 0xBF80, 0x4000, 0x0000, 0x8000], dtype=np.uint16)  # 1, -1, 2, +0, -0
    h = oracle.gelu_bf16(y)
    assert [hex(v) for v in h[:3]] == ["0x3f57", "0xbe22", "0x3ffa"]
    assert h[3] == 0x0000 and h[4] in (0x0000, 0x8000)  # GELU(-0) = -0 * 1/2


# --- static per-tensor E4M3 activations -------------------------------------------------------
#
# codes = RNE_sat(x / s) on the E4M3 grid, x / s the exact quotient; the linear multiplies its
# sums by s.  Pinned against exact rationals (tests/_exact.py), never against binary32
# arithmetic.

def _f32(v: float) -> float:
    return float(np.float32(v))


@pytest.mark.parametrize("scale", [0.5, 0.0371, 2.0 ** -7 * 3, 11.0, 7.3e-31, 3.1e29])
def test_static_e4m3_is_nearest_grid_point_of_the_exact_quotient(scale):
    """Each code is the E4M3 value nearest to the exact rational x / s (ties to the even
    code, saturating, sign kept), found by exact comparison with every grid neighbour."""
    s = _f32(scale)
    rng = np.random.default_rng(int(abs(np.log2(s))) + 3)
    x = (rng.standard_normal(3000) * s * rng.choice([1.0, 30.0, 300.0, 1e-3, 1e-6], size=3000)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)          # truncate to bf16 (any bf16 will do)
    got = oracle.quantize_static_e4m3(bits, s)
    S = _exact.f32_fraction(s)
    for b, c in zip(bits, got):
        xf = _exact.bf16_fraction(int(b))
        want = _exact.nearest_code(xf / S, oracle.E4M3, negative=bool(b & 0x8000))
        assert c == want, (hex(int(b)), s, hex(c), hex(want))


def test_static_e4m3_near_ties_follow_the_exact_quotient():
    """Inputs for which a binary32 evaluation of x / s -- the correctly rounded binary32
    quotient (double rounding) or the binary32 product x * fl32(1/s) -- takes another code
    than the exact quotient: the oracle takes the exact quotient's code, for x scaled by
    powers of two across the E4M3 range and for both signs."""
    cases = _exact.static_near_ties()
    assert len(cases) > 400
    checked = 0
    for s, x in cases[::3]:
        sf = float(s)
        xs = [x * Fraction(2) ** j for j in range(-6, 9)]
        xs = [v for v in xs if Fraction(2) ** -9 <= v / s <= 448]
        bits = np.array([_exact.bf16_bits(v) for v in xs] + [_exact.bf16_bits(v) | 0x8000 for v in xs],
                        dtype=np.uint16)
        got = oracle.quantize_static_e4m3(bits, sf)
        for b, c in zip(bits, got):
            want = _exact.nearest_code(_exact.bf16_fraction(int(b)) / s, oracle.E4M3)
            assert c == want, (hex(int(b)), s, hex(c), hex(want))
            checked += 1
    assert checked > 2000


def test_static_e4m3_exact_multiples_saturation_and_sign():
    s = 2.0 ** -3  # x = q * s is exact for every E4M3 value q, and so is x / s
    qs = [oracle.decode_elem(c, oracle.E4M3) for c in range(0x7F)]  # every non-negative finite code
    xb = np.array([oracle.double_to_bf16(q * s) for q in qs], dtype=np.uint16)
    assert list(oracle.quantize_static_e4m3(xb, s)) == list(range(0x7F))
    big = np.array([oracle.double_to_bf16(v) for v in (449 * s, 1e4 * s, -1e4 * s, -1e-9, 1e-9)], dtype=np.uint16)
    assert [hex(c) for c in oracle.quantize_static_e4m3(big, s)] == ["0x7e", "0x7e", "0xfe", "0x80", "0x0"]


def test_linear_scaled_brute_force_exact():
    """alpha * sum_k deq(a) * deq(w) + bias, checked with exact rationals."""
    rng = np.random.default_rng(21)
    M, N, K = 3, 4, 64
    a_codes = rng.integers(0, 256, size=(M, K), dtype=np.uint8)
    a_codes[(a_codes & 0x7F) == 0x7F] = 0x11  # no NaN codes
    a_sf = np.full((M, K // 32), 127, dtype=np.uint8)
    w_codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    w_sf = rng.integers(120, 135, size=(N, K // 32), dtype=np.uint8)
    bias = np.array([oracle.double_to_bf16(v) for v in (0.5, -1.25, 3.0, 0.0)], dtype=np.uint16)
    alpha = 0.1234567
    y = oracle.linear_rows_scaled(a_codes, a_sf, oracle.E4M3, np.arange(M), K, w_codes, w_sf, alpha, bias)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                wc = (int(w_codes[n, k // 2]) >> (4 * (k & 1))) & 0xF
                acc += (Fraction(oracle.decode_elem(int(a_codes[m, k]), oracle.E4M3)) *
                        Fraction(oracle.decode_elem(wc, oracle.E2M1)) * Fraction(2) ** (int(w_sf[n, k // 32]) - 127))
            want = Fraction(alpha) * acc + Fraction(oracle.bf16_to_float(int(bias[n])))
            assert abs(Fraction(y[m, n]) - want) <= abs(want) * Fraction(1, 10 ** 14) + Fraction(1, 10 ** 300)


# --- transform_on: smoothing and block Hadamard rotation ------------------------------------
#
# Definition: t = (x * mul) . blockdiag(H_B) / sqrt(B), then MX quantization of t.  Pinned
# against exact rationals: the transformed values are S / sqrt(B) with S an exact sum, and
# every scale and code decision compares squares exactly (tests/_exact.py).

def _bf16_bits(a):
    return (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _unpack_codes(codes, K, fmt):
    if fmt == oracle.E4M3:
        return codes.reshape(-1, K)
    lo, hi = codes & 0xF, codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(-1, K)


@pytest.mark.parametrize("B", [32, 128])
@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
@pytest.mark.parametrize("smooth", [False, True])
def test_transform_matches_exact_rationals(B, fmt, smooth):
    """Scales and codes of the definition on random rows with an outlier channel, every
    one decided by exact rational comparisons."""
    f = FMT[fmt]
    emax = 2 if f == oracle.E2M1 else 8
    rng = np.random.default_rng(B + 7 * f + int(smooth))
    M, K = 3, 256
    x = rng.standard_normal((M, K)) * 3.0
    x[:, 5] *= 60.0
    x[1, 40:72] *= 1e-3
    bits = _bf16_bits(x)
    mul = rng.uniform(0.25, 4.0, size=K).astype(np.float32) if smooth else None
    o = oracle.quantize_transformed(bits, f, B, mul)
    got_codes = _unpack_codes(o["codes"], K, f)
    for r in range(M):
        S = _exact.transform_exact(bits[r], B, mul)
        for kb in range(K // 32):
            blk = S[kb * 32:(kb + 1) * 32]
            sc = _exact.scale_code_sqrt(blk, B, emax)
            assert o["sf"][r, kb] == sc, (r, kb, o["sf"][r, kb], sc)
            X = Fraction(2) ** (sc - 127)
            for i, v in enumerate(blk):
                want = _exact.nearest_code_sqrt(v, B, X, f)
                assert got_codes[r, kb * 32 + i] == want, (r, kb, i, got_codes[r, kb * 32 + i], want)


def _near_boundary_row(B, target):
    """A row whose first rotation block is [x0, x1, x2, x3, 0, ...] with x0 + x1 + x2 + x3
    equal to target to about 32 bits (four bf16 values taking 8 bits each), so that output
    0 of the rotation, (x0 + .. + x3) / sqrt(B), lands within about 2^-30 of target / sqrt(B)."""
    xs, rest = [], Fraction(target)
    for _ in range(4):
        b = int(_bf16_bits([float(rest)])[0])
        xs.append(b)
        rest -= _exact.bf16_fraction(b)
    row = np.zeros(B, dtype=np.uint16)
    row[:4] = xs
    return row


def test_transform_flags_values_near_a_grid_midpoint():
    """Output 0 placed within 2^-30 (relative) of the E2M1 midpoint 5 (between 4 and 6) at
    scale 1: a binary32 evaluation could round it either way, so the oracle reports two
    candidate codes; its own code is the exact value's."""
    import math
    B = 32
    for side in (-1, 1):
        target = Fraction(5) * Fraction(math.sqrt(B)) * (1 + side * Fraction(1, 2 ** 31))
        row = _near_boundary_row(B, target)
        o = oracle.quantize_transformed(row[None, :], oracle.E2M1, B)
        S = _exact.transform_exact(row, B)
        sc = _exact.scale_code_sqrt(S[:32], B, 2)
        assert o["sf"][0, 0] == sc == 127
        want = _exact.nearest_code_sqrt(S[0], B, Fraction(1), oracle.E2M1)
        assert _unpack_codes(o["codes"], B, oracle.E2M1)[0, 0] == want
        assert {o["code_lo"][0, 0], o["code_hi"][0, 0]} == {6, 7}          # 4 or 6
        assert (o["code_lo"][0, 1:] == o["code_hi"][0, 1:]).sum() >= 24  # the others mostly certain


def test_transform_flags_a_scale_near_a_power_of_two():
    """A block whose largest transformed value is within 2^-30 of 8: floor(log2) is 2 or 3
    depending on rounding, so the block's scale is flagged; a block well inside a binade
    is not."""
    import math
    B = 32
    row = _near_boundary_row(B, Fraction(8) * Fraction(math.sqrt(B)) * (1 - Fraction(1, 2 ** 31)))
    o = oracle.quantize_transformed(row[None, :], oracle.E2M1, B)
    assert o["blk_amb"][0, 0] == 1
    row2 = _near_boundary_row(B, Fraction(11) * Fraction(math.sqrt(B)))
    o2 = oracle.quantize_transformed(row2[None, :], oracle.E2M1, B)
    assert o2["blk_amb"][0, 0] == 0


def test_transform_flags_possible_binary32_overflow():
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, :4] = 2.0 ** 126
    o = oracle.quantize_transformed(_bf16_bits(x), oracle.E4M3, 32)
    assert o["blk_amb"][0, 0] == 2
    assert o["sf"][0, 0] != 255        # the definition's block is finite (t = 2^126 * 4 / sqrt 32)


@pytest.mark.parametrize("B", [32, 128])
def test_transform_is_scaled_hadamard_rotation(B):
    """t equals (x * mul) . blockdiag(H_B) / sqrt(B) with scipy's Sylvester matrix in fp64 to
    fp64 rounding; codes and scales dequantize to within one element step of t."""
    from scipy.linalg import hadamard
    rng = np.random.default_rng(B + 1)
    M, K = 6, 256
    x = (rng.standard_normal((M, K)) * 3).astype(np.float32)
    x[:, 5] *= 60.0
    bits = _bf16_bits(x)
    xb = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mul = rng.uniform(0.5, 2.0, size=K).astype(np.float32)
    o = oracle.quantize_transformed(bits, oracle.E2M1, B, mul)
    H = hadamard(B).astype(np.float64) / np.sqrt(B)
    want = np.concatenate([(xb * mul.astype(np.float64))[:, b0:b0 + B] @ H for b0 in range(0, K, B)], axis=1)
    assert np.abs(o["t"] - want).max() <= 1e-13 * np.abs(want).max()
    deq = oracle.dequantize(o["codes"], o["sf"], K, oracle.E2M1)
    scale = np.repeat(2.0 ** (o["sf"].astype(np.float64) - 127), 32, axis=1)
    assert (np.abs(deq - o["t"]) <= 2.0 * scale + 1e-30).all()   # within the largest E2M1 step (4 -> 6)


def test_transform_power_of_two_smoothing_shifts_only_the_scales():
    """A smoothing multiplier of 2^j on every channel scales the transformed values exactly,
    so the element codes are unchanged and every scale code moves by j."""
    rng = np.random.default_rng(9)
    bits = _bf16_bits(rng.standard_normal((4, 128)) * 2)
    o0 = oracle.quantize_transformed(bits, oracle.E4M3, 32, None)
    o1 = oracle.quantize_transformed(bits, oracle.E4M3, 32, np.full(128, 8.0, dtype=np.float32))
    assert np.array_equal(o0["codes"], o1["codes"])
    assert np.array_equal(o1["sf"].astype(int), o0["sf"].astype(int) + 3)


def test_transform_sign_symmetry():
    rng = np.random.default_rng(10)
    bits = _bf16_bits(rng.standard_normal((3, 128)))
    o0 = oracle.quantize_transformed(bits, oracle.E4M3, 128, None)
    o1 = oracle.quantize_transformed(bits ^ 0x8000, oracle.E4M3, 128, None)
    assert np.array_equal(o1["t"], -o0["t"]) and np.array_equal(o0["sf"], o1["sf"])
    nz = o0["t"] != 0
    assert np.array_equal(o1["codes"][nz], o0["codes"][nz] ^ 0x80)


# --- SVDQuant low-rank branch ------------------------------------------------------------------

def _lowrank_case(rng, M, N, K, r):
    a_codes = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    a_sf = rng.integers(120, 132, size=(M, K // 32), dtype=np.uint8)
    r_codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    r_sf = rng.integers(120, 132, size=(N, K // 32), dtype=np.uint8)
    bf = lambda a: (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)  # noqa: E731
    x = bf(rng.standard_normal((M, K)))
    l1t = bf(rng.standard_normal((r, K)) * 0.1)
    l2t = bf(rng.standard_normal((N, r)) * 0.1)
    bias = bf(rng.standard_normal(N))
    return a_codes, a_sf, r_codes, r_sf, x, l1t, l2t, bias


def test_lowrank_with_zero_branch_is_the_linear():
    rng = np.random.default_rng(31)
    M, N, K, r = 5, 7, 64, 16
    a_codes, a_sf, r_codes, r_sf, x, l1t, l2t, bias = _lowrank_case(rng, M, N, K, r)
    zero = np.zeros_like(l1t)
    y = oracle.linear_lowrank_rows(a_codes, a_sf, oracle.E2M1, np.arange(M), K, r_codes, r_sf, x, zero, l2t, bias)
    want = oracle.linear_rows(a_codes, a_sf, oracle.E2M1, np.arange(M), K, r_codes, r_sf, bias)
    assert np.array_equal(y, want)


def test_lowrank_brute_force_exact():
    """Exact rationals: the quantized product, the bf16-rounded branch activation u (its
    rounding checked against the pinned bf16 rounding) times l2t, and the bias."""
    rng = np.random.default_rng(32)
    M, N, K, r = 2, 3, 32, 4
    a_codes, a_sf, r_codes, r_sf, x, l1t, l2t, bias = _lowrank_case(rng, M, N, K, r)
    y = oracle.linear_lowrank_rows(a_codes, a_sf, oracle.E2M1, np.arange(M), K, r_codes, r_sf, x, l1t, l2t, bias)
    f = lambda b: Fraction(oracle.bf16_to_float(int(b)))  # noqa: E731
    for m in range(M):
        u = []
        for j in range(r):
            exact = sum(f(x[m, k]) * f(l1t[j, k]) for k in range(K))
            u.append(f(oracle.double_to_bf16(float(exact))))
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                ac = (int(a_codes[m, k // 2]) >> (4 * (k & 1))) & 0xF
                rc = (int(r_codes[n, k // 2]) >> (4 * (k & 1))) & 0xF
                acc += (Fraction(oracle.decode_elem(ac, oracle.E2M1)) * Fraction(2) ** (int(a_sf[m, k // 32]) - 127) *
                        Fraction(oracle.decode_elem(rc, oracle.E2M1)) * Fraction(2) ** (int(r_sf[n, k // 32]) - 127))
            want = acc + sum(u[j] * f(l2t[n, j]) for j in range(r)) + f(bias[n])
            assert abs(Fraction(y[m, n]) - want) <= abs(want) * Fraction(1, 10 ** 13) + Fraction(1, 10 ** 300)


# --- the bf16 GEMM and the policy's calibration arithmetic ----------------------------------

def test_gemm_bf16_brute_force_exact():
    rng = np.random.default_rng(41)
    M, N, K = 3, 4, 24
    a = _bf16_bits(rng.standard_normal((M, K)))
    b = _bf16_bits(rng.standard_normal((N, K)) * 0.1)
    bias = _bf16_bits(rng.standard_normal(N))
    y = oracle.gemm_bf16(a, b, bias)
    f = lambda v: _exact.bf16_fraction(int(v))  # noqa: E731
    for m in range(M):
        for n in range(N):
            want = sum(f(a[m, k]) * f(b[n, k]) for k in range(K)) + f(bias[n])
            assert abs(Fraction(y[m, n]) - want) <= abs(want) * Fraction(1, 10 ** 14)


def test_channel_absmax_hand_values():
    x = np.array([[1.0, -2.0, 0.0, 3.5], [-4.0, 1.5, -0.0, -3.5]], dtype=np.float32)
    assert list(oracle.channel_absmax(_bf16_bits(x))) == [4.0, 2.0, 0.0, 3.5]


def test_smooth_scales_closed_forms():
    ax = np.array([4.0, 9.0, 0.0, 1e-9])
    aw = np.array([1.0, 0.25, 2.0, 16.0])
    # alpha = 1: s = max|X|; alpha = 0: s = 1 / max|W|; alpha = 1/2: sqrt(max|X| / max|W|)
    f = float(np.float32(1e-5))
    assert np.allclose(oracle.smooth_scales(ax, aw, 1.0), [4.0, 9.0, f, f], rtol=0, atol=0)
    assert np.allclose(oracle.smooth_scales(ax, aw, 0.0), [1.0, 4.0, 0.5, 1 / 16.0], rtol=1e-15)
    assert np.allclose(oracle.smooth_scales(ax, aw, 0.5), [2.0, 6.0, np.sqrt(f / 2.0), np.sqrt(f / 16.0)], rtol=1e-15)
    # scaling the activation's channel maxima by c scales s by c^alpha
    s1 = oracle.smooth_scales(ax[:2] * 16.0, aw[:2], 0.25)
    assert np.allclose(s1, 2.0 * oracle.smooth_scales(ax[:2], aw[:2], 0.25), rtol=1e-15)


def test_sqnr_known_ratio():
    """test = ref * (1 + 2^-7) exactly: every error is ref * 2^-7, so the ratio of the sums is
    2^14 and the SQNR 140 log10(2) dB; split over two tensors it is the same."""
    ref = _bf16_bits(np.full(64, 2.0))
    test = _bf16_bits(np.full(64, 2.0 * (1 + 2.0 ** -7)))
    num, den, db = oracle.sqnr([ref], [test])
    assert num == 64 * 4.0 and den == 64 * 4.0 * 2.0 ** -14
    assert abs(db - 140 * math.log10(2.0)) < 1e-12
    assert oracle.sqnr([ref[:32], ref[32:]], [test[:32], test[32:]])[2] == db


def test_lowrank_split_exact_recomposition():
    """Singular vectors and values chosen so that U sqrt(S) and sqrt(S) Vh are bf16 values
    (S powers of 4): the factors are those products exactly, and W built as l2t . l1t + R with
    a bf16 R whose sum is exact returns R as the residual."""
    rng = np.random.default_rng(5)
    N, K, r = 6, 40, 3
    U = _bf16_f32(rng.standard_normal((N, r)))
    Vh = _bf16_f32(rng.standard_normal((r, K)))
    S = np.array([16.0, 4.0, 0.25], dtype=np.float32)
    l2t_v = U.astype(np.float64) * np.sqrt(S)[None, :]
    l1t_v = np.sqrt(S)[:, None] * Vh.astype(np.float64)
    R = _bf16_f32(rng.standard_normal((N, K)) * 2.0 ** -20)
    W = l2t_v @ l1t_v + R
    w_bits = oracle.round_bf16(W)
    l1t, l2t, resid = oracle.lowrank_split(U, S, Vh, w_bits, r)
    assert np.array_equal(oracle.bf16_bits_to_f64(l2t), l2t_v)
    assert np.array_equal(oracle.bf16_bits_to_f64(l1t), l1t_v)
    want = oracle.round_bf16(oracle.bf16_bits_to_f64(w_bits) - l2t_v @ l1t_v)
    assert np.array_equal(resid, want)
    # rank 0 leaves the weight itself
    assert np.array_equal(oracle.lowrank_split(U, S, Vh, w_bits, 0)[2], w_bits)


def _bf16_f32(a):
    return oracle.bf16_bits_to_f64(_bf16_bits(a)).astype(np.float32)
