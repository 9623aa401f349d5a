"""The NVFP4 dequantization arithmetic of the GPU kernels, checked on the CPU
against the E2M1 / E4M3 definitions (NVFP4 storage of the Nemotron-H
checkpoint: vllm.cpp PR #518, row spec).

The kernels build each weight without the conversion pipe: two 4-bit codes
placed in the low bytes of the two 16-bit halves of a word p are turned into
two bf16 bit patterns by one integer multiply and one mask,
``(p * (2^6 + 2^12)) & 0x81C081C0``, which read as ``code * 2^-126`` (code
0.5 as the bf16 subnormal 2^-127).  One bf16 multiply by ``scale * 2^118``
then gives ``code * scale * 2^-8``; these tests check that both steps are
exact for every code and every finite scale byte, with plain integer and
rational arithmetic (no GPU, no float rounding to hide behind).
"""
from fractions import Fraction

MULT = (1 << 6) + (1 << 12)
MASK = 0x81C081C0


def e2m1(code):
    """E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit."""
    sign = -1 if code & 8 else 1
    e, m = (code >> 1) & 3, code & 1
    mag = Fraction(m, 2) if e == 0 else Fraction(2) ** (e - 1) * (1 + Fraction(m, 2))
    return sign * mag


def e4m3(byte):
    """E4M3 (bias 7, no infinities); None for NaN (S.1111.111)."""
    e, m = (byte >> 3) & 15, byte & 7
    if e == 15 and m == 7:
        return None
    sign = -1 if byte & 0x80 else 1
    mag = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return sign * mag


def bf16(bits):
    """Exact value of a bf16 bit pattern (finite patterns only)."""
    sign = -1 if bits & 0x8000 else 1
    e, m = (bits >> 7) & 0xFF, bits & 0x7F
    assert e != 0xFF
    if e == 0:
        return sign * Fraction(m, 128) * Fraction(2) ** -126
    return sign * (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)


def bf16_exact(v):
    """The bf16 pattern of v when v is exactly representable (else None)."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    if e < -126 or e > 127:
        return None
    frac = (a - 1) * 128
    if frac.denominator != 1:
        return None
    return sign | ((e + 127) << 7) | int(frac)


def test_every_code_pair_reads_as_code_times_2_pow_minus_126():
    for lo in range(16):
        for hi in range(16):
            p = lo | (hi << 16)
            bits = (p * MULT) & MASK
            assert p * MULT < 1 << 32                       # no carry out of the word
            assert bf16(bits & 0xFFFF) == e2m1(lo) * Fraction(2) ** -126, (lo, hi)
            assert bf16(bits >> 16) == e2m1(hi) * Fraction(2) ** -126, (lo, hi)


def test_scale_multiplier_and_product_are_exact():
    codes = [e2m1(c) for c in range(16)]
    n = 0
    for byte in range(128):                                # the scales are non-negative
        s = e4m3(byte)
        if s is None:
            continue
        mult = bf16_exact(s * Fraction(2) ** 118)
        assert mult is not None, byte                      # scale * 2^118 is a bf16 value
        for c in codes:
            prod = c * Fraction(2) ** -126 * bf16(mult)
            assert prod == c * s * Fraction(2) ** -8
            assert bf16_exact(prod) is not None, (c, byte)  # the bf16 multiply rounds nothing
        n += 1
    assert n == 127                                        # every finite scale byte
