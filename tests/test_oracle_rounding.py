"""Pins for two roundings every GPU bit-exactness claim rests on:

* the oracle's fp32 -> bf16 conversion (the rounding of every matmul operand
  and of the bf16 dequantised weight; reading R6: round to nearest, ties to
  even), and
* the operation order of double quantisation ("QLoRA explained", section
  "Double quantization": the scale divided by the group constant, then times
  127, rounded to an integer; the dequantised scale is the code times
  fl32(c_g / 127)), as opposed to the other order printed in "Parameter-
  Efficient Fine-Tuning", section "Vanilla Uniform Quantization" (a factor
  127 / absmax applied to the value).

The expected values are computed here from the definitions with exact
rationals (fractions.Fraction) and an explicit IEEE rounding step written from
the definition of a binary floating-point format. The cases are chosen so
that the competing readings give different answers: truncating to bf16,
rounding ties away from zero, or swapping either double-quant order makes a
test here fail.
"""
from fractions import Fraction

import numpy as np

import oracle

# --------------------------------------------------------------------------
# exact rounding to a binary format, from the definition
# --------------------------------------------------------------------------
INF = object()     # marker for an overflow to infinity


def round_to_format(x: Fraction, prec: int, emin: int, emax: int):
    """Round x to the nearest number with `prec` significant bits, exponent in
    [emin, emax] (subnormals below 2^emin), ties to the even significand.
    Returns a Fraction, or (sign, INF) on overflow."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    # exponent e with 2^e <= a < 2^(e+1), found exactly
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)                         # subnormal range keeps the spacing of 2^emin
    ulp = Fraction(2) ** (e - prec + 1)
    q = a / ulp
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * ulp
    if r >= Fraction(2) ** (emax + 1):
        return (sign, INF)
    return sign * r


def fl32(x: Fraction) -> Fraction:
    r = round_to_format(x, 24, -126, 127)
    assert not isinstance(r, tuple), "no fp32 overflow expected here"
    return r


def rne_int(x: Fraction) -> int:
    """Nearest integer, ties to even."""
    n = x.numerator // x.denominator
    rem = x - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def frac32(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def f32_of(x: Fraction) -> np.float32:
    v = np.float32(float(x))
    assert Fraction(float(v)) == x
    return v


# --------------------------------------------------------------------------
# fp32 -> bf16, round to nearest even
# --------------------------------------------------------------------------
def expected_bf16_bits(v: np.float32) -> int:
    u = int(np.array(v, dtype=np.float32).view(np.uint32))
    if (u & 0x7F800000) == 0x7F800000:
        if u & 0x007FFFFF:
            return -1                      # NaN: any NaN pattern is accepted
        return u >> 16                     # infinities are kept
    r = round_to_format(Fraction(float(v)), 8, -126, 127)
    if isinstance(r, tuple):
        return 0xFF80 if r[0] < 0 else 0x7F80
    if r == 0:
        return (u >> 16) & 0x8000          # the sign of zero is kept
    bits = int(np.array(np.float32(float(r)), dtype=np.float32).view(np.uint32))
    assert bits & 0xFFFF == 0
    return bits >> 16


def check_bf16(vals):
    vals = np.asarray(vals, dtype=np.float32)
    got = oracle.f32_to_bf16(vals)
    for v, g in zip(vals, got):
        want = expected_bf16_bits(v)
        if want < 0:
            assert (int(g) & 0x7F80) == 0x7F80 and (int(g) & 0x7F) != 0, (v, hex(int(g)))
        else:
            assert int(g) == want, (float(v), hex(int(g)), hex(want))


def f32(bits: int) -> np.float32:
    return np.array(bits, dtype=np.uint32).view(np.float32)[()]


def test_bf16_half_ulp_ties_go_to_even():
    # bf16 keeps 7 fraction bits: at 1.0 the spacing is 2^-7, half of it 2^-8
    one = Fraction(1)
    h = Fraction(1, 2 ** 8)
    cases = {
        one + h: one,                          # tie between 1 (even) and 1 + 2^-7 (odd)
        one + 3 * h: one + 4 * h,              # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
        -(one + h): -one,
        -(one + 3 * h): -(one + 4 * h),
        Fraction(3, 2) + h: Fraction(3, 2),    # 1.5 has an even last bit
    }
    for x, want in cases.items():
        got = oracle.f32_to_bf16(np.array([f32_of(x)], dtype=np.float32))[0]
        assert Fraction(float(oracle.bf16_to_f64(np.array([got]))[0])) == want, float(x)
    check_bf16([f32_of(x) for x in cases])


def test_bf16_just_below_and_above_a_tie():
    ties = [f32_of(Fraction(1) + Fraction(2 * k + 1, 2 ** 8)) for k in range(8)]
    below = [np.nextafter(t, np.float32(0)) for t in ties]
    above = [np.nextafter(t, np.float32(2)) for t in ties]
    check_bf16(ties + below + above)
    # the value one fp32 ulp below the first tie rounds down, one above rounds up
    lo = oracle.f32_to_bf16(np.array([below[0], above[0]], dtype=np.float32))
    assert list(lo) == [0x3F80, 0x3F81]


def test_bf16_overflow_subnormals_zero_nan_inf():
    big = [f32(0x7F7FFFFF), f32(0x7F7F8000), f32(0x7F7F7FFF), f32(0xFF7FFFFF), f32(0x7F7F0000)]
    sub = [f32(0x00000001), f32(0x00008000), f32(0x00018000), f32(0x00007FFF), f32(0x80008001),
           f32(0x007FFFFF), f32(0x00800000)]
    special = [np.float32(0.0), np.float32(-0.0), np.float32(np.inf), np.float32(-np.inf),
               f32(0x7FC00000), f32(0x7F800001), f32(0xFFFFFFFF)]
    check_bf16(big + sub + special)
    got = oracle.f32_to_bf16(np.array([big[0], big[1], big[2]], dtype=np.float32))
    assert list(got) == [0x7F80, 0x7F80, 0x7F7F]      # the largest finite fp32 rounds to +inf


def test_bf16_random_bit_patterns():
    rng = np.random.default_rng(2024)
    u = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    # half of them with the low 16 bits forced to an exact tie or a near-tie
    u[::2] = (u[::2] & 0xFFFF0000) | rng.choice([0x8000, 0x7FFF, 0x8001], size=u[::2].size)
    vals = u.view(np.float32)
    finite = vals[np.isfinite(vals)]
    check_bf16(finite)


# --------------------------------------------------------------------------
# double-quant operation order
# --------------------------------------------------------------------------
def q8_stated(s: Fraction, c: Fraction) -> int:
    """RNE(fl32(fl32(s / c) * 127)): divide by the group constant, then scale."""
    return rne_int(fl32(fl32(s / c) * 127))


def q8_swapped(s: Fraction, c: Fraction) -> int:
    """The other order: a factor fl32(127 / c) applied to s."""
    return rne_int(fl32(fl32(Fraction(127) / c) * s))


def shat_stated(q: int, c: Fraction) -> Fraction:
    """fl32(q8 * fl32(c / 127))."""
    return fl32(q * fl32(c / 127))


def shat_swapped(q: int, c: Fraction) -> Fraction:
    """fl32(fl32(q8 * c) / 127)."""
    return fl32(fl32(q * c) / 127)


def discriminating_scales(c: Fraction, want: int = 24):
    """Block maxima s <= c on which the two q8 orders disagree: fp32 values a few
    ulps around (j + 1/2) c / 127 for every code j."""
    found = []
    for j in range(127):
        s0 = np.float32(float(fl32((j + Fraction(1, 2)) * c / 127)))
        cands = [s0]
        lo = hi = s0
        for _ in range(6):
            lo = np.nextafter(lo, np.float32(0))
            hi = np.nextafter(hi, np.float32(np.inf))
            cands += [lo, hi]
        for v in cands:
            s = Fraction(float(v))
            if 0 < s <= c and q8_stated(s, c) != q8_swapped(s, c):
                found.append(v)
                break
        if len(found) >= want:
            break
    return found


def test_double_quant_code_order_pinned():
    rng = np.random.default_rng(31)
    group_consts = [np.float32(v) for v in (0.7391234, 0.0123457, 3.14159, 1e-3 * 1.2345678,
                                            rng.uniform(0.01, 0.1))]
    blocks, expect, total_disc = [], [], 0
    for c32 in group_consts:
        c = Fraction(float(c32))
        disc = discriminating_scales(c)
        total_disc += len(disc)
        # one group of 256 blocks: its maximum c first, then the discriminating
        # maxima, then random maxima in (0, c]
        rest = [np.float32(v) for v in rng.uniform(0, float(c32), size=255 - len(disc))]
        maxima = [c32] + disc + rest
        for s in maxima:
            b = np.zeros(64, dtype=np.float32)
            b[int(rng.integers(0, 64))] = -s if rng.random() < 0.5 else s
            blocks.append(b)
            expect.append(q8_stated(Fraction(float(s)), c))
    assert total_disc >= 40, "the pin needs inputs on which the two orders differ"
    q = oracle.quantize(np.concatenate(blocks), dq=True)
    assert list(q.cg) == group_consts
    assert [int(v) for v in q.q8] == expect
    swapped = [q8_swapped(Fraction(float(s)), Fraction(float(group_consts[i // 256])))
               for i, s in enumerate(q.absmax)]
    assert sum(a != b for a, b in zip(swapped, expect)) >= 40


def test_double_quant_scale_order_pinned():
    rng = np.random.default_rng(32)
    group_consts = [np.float32(v) for v in rng.uniform(1e-3, 2.0, size=6)]
    blocks = []
    for c32 in group_consts:
        maxima = [c32] + [np.float32(v) for v in rng.uniform(0, float(c32), size=255)]
        for s in maxima:
            b = np.zeros(64, dtype=np.float32)
            b[0] = s
            blocks.append(b)
    q = oracle.quantize(np.concatenate(blocks), dq=True)
    got = oracle.block_scales(q)
    differ = 0
    for i, (qq, g) in enumerate(zip(q.q8, got)):
        c = Fraction(float(q.cg[i // 256]))
        want = shat_stated(int(qq), c)
        assert Fraction(float(g)) == want, (i, int(qq), float(g), float(want))
        differ += want != shat_swapped(int(qq), c)
    assert differ >= 100, "the pin needs codes on which the two orders differ"


def test_exact_rounding_helper_against_ieee_single_operations():
    """The helper agrees with IEEE fp32 division and multiplication (numpy's
    float32 arithmetic is one correctly rounded operation each), so the
    expectations above use the same fp32 rounding the definition asks for."""
    rng = np.random.default_rng(33)
    a = rng.uniform(-4, 4, 3000).astype(np.float32)
    b = rng.uniform(0.01, 4, 3000).astype(np.float32)
    with np.errstate(all="ignore"):
        qd = a / b
        qm = a * b
    for x, y, d, m in zip(a, b, qd, qm):
        assert fl32(frac32(x) / frac32(y)) == frac32(d)
        assert fl32(frac32(x) * frac32(y)) == frac32(m)
