"""The fp16 arithmetic identities the CUDA kernels' in-register unpack relies on, checked
exhaustively on the CPU with numpy's binary16 rounding (a fused multiply-add is emulated as the
exact fp64 value rounded once to fp16; every operand here is an fp16 value, so the fp64 product
plus addend is exact).  The expected values are the containers' definitions: a PQ2_0 field holds
code + 1 in two bits; a PTQ1_0 quintet byte holds five base-3 digits code + 1, least significant
first ("Scion-35B-A3B" and "Scion-FlashNext-176B-A6B" model cards, Weight Representation).
"""
import numpy as np
import pytest


def f16(v):
    return np.asarray(v, np.float64).astype(np.float16)


def bits_to_f64(b):
    return np.asarray(b, np.uint16).view(np.float16).astype(np.float64)


def fma16(a, b, c):
    return f16(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


HALVES = np.arange(1 << 16, dtype=np.uint32)


@pytest.mark.parametrize("s", range(8))
def test_pq2_subnormal_fields(s):
    """Decode ring kernels: pair s takes the field at bits 2f..2f+1 (f = s, or s - 5 after a
    10-bit shift); masked alone it is the fp16 subnormal b * 4^f * 2^-24 with b the stored field."""
    f = s if s < 5 else s - 5
    src = HALVES if s < 5 else HALVES >> 10
    b = (src >> (2 * f)) & 3
    masked = src & (3 << (2 * f))
    np.testing.assert_array_equal(bits_to_f64(masked), b * 4.0 ** f * 2.0 ** -24)


@pytest.mark.parametrize("s", range(8))
def test_pq2_magic_fields(s):
    """Split-K decode expansion: the field ORed into the fp16 pattern of 1024, minus 1024 + 4^f,
    is 4^f * (b - 1) = 4^f * code, with no rounding."""
    f = s if s < 5 else s - 5
    src = HALVES if s < 5 else HALVES >> 10
    b = (src >> (2 * f)) & 3
    v = bits_to_f64((src & (3 << (2 * f))) | 0x6400)
    got = f16(v.astype(np.float16).astype(np.float64) - f16(1024 + 4 ** f).astype(np.float64))
    np.testing.assert_array_equal(got.astype(np.float64), 4.0 ** f * (b.astype(np.float64) - 1))


@pytest.mark.parametrize("s", range(8))
def test_pq2_exponent_magic_fields(s):
    """Prefill expansion: the field at bits 2f..2f+1 ORed into the fp16 pattern with exponent
    field 25 - 2f (the value 2^(10-2f), whose mantissa unit is 4^-f) reads 2^(10-2f) + b; minus
    2^(10-2f) + 1 (that pattern with bit 2f set) it is the code b - 1, with no rounding and no
    position factor."""
    f = s if s < 5 else s - 5
    src = HALVES if s < 5 else HALVES >> 10
    b = ((src >> (2 * f)) & 3).astype(np.float64)
    magic = (25 - 2 * f) << 10
    v = bits_to_f64((src & (3 << (2 * f))) | magic)
    np.testing.assert_array_equal(v, 2.0 ** (10 - 2 * f) + b)
    bias = float(bits_to_f64(magic | (1 << (2 * f))))
    assert bias == 2.0 ** (10 - 2 * f) + 1
    np.testing.assert_array_equal(f16(v - bias).astype(np.float64), b - 1)


def test_pq2_scaled_expansion_exact():
    """Prefill expansion: code times an fp16 group scale is exact in fp16 for every finite fp16
    scale (the product is the scale, zero or its negation)."""
    scales = np.arange(1 << 16, dtype=np.uint16).view(np.float16)
    scales = scales[np.isfinite(scales)].astype(np.float64)
    for code in (-1.0, 0.0, 1.0):
        got = f16(f16(code).astype(np.float64) * scales)
        np.testing.assert_array_equal(got.astype(np.float64), code * scales)


def _digit_chain(V, n):
    """n steps of the kernels' base-3 chain on fp16 values V = 1024 + v."""
    third, c1, m3, c2047 = f16(0.333251953125), f16(682.5), f16(-3.0), f16(2047.0)
    out = []
    for _ in range(n):
        Vn = fma16(V, third, c1)
        code = f16(fma16(Vn, m3, V).astype(np.float64) + c2047.astype(np.float64))
        out.append(code.astype(np.float64))
        V = Vn
    return out


def test_ptq1_digit_chain_all_quintets():
    """Every valid quintet byte (0..242): the chain yields its five digits minus one, least
    significant first."""
    v = np.arange(243)
    codes = _digit_chain(f16(1024 + v), 5)
    for j in range(5):
        np.testing.assert_array_equal(codes[j], (v // 3 ** j) % 3 - 1)


def test_ptq1_digit_chain_tail_byte():
    """The tail byte (0..26) holds three digits; the same chain reads them."""
    v = np.arange(27)
    codes = _digit_chain(f16(1024 + v), 3)
    for j in range(3):
        np.testing.assert_array_equal(codes[j], (v // 3 ** j) % 3 - 1)


def test_ptq1_chain_constants_are_fp16():
    """The chain's constants are exact fp16 values (no rounding when they are loaded)."""
    for c in (0.333251953125, 682.5, -3.0, 2047.0):
        assert float(f16(c)) == c


def test_ptq1_remainder_fields_all_bytes():
    """The eight remainder trits of a row (digits 0..4 of quintet byte 24, 0..2 of the tail byte)
    re-encoded as 2-bit fields, even trits in one byte and odd trits in the other, are read back
    by lane-column c as the fp16 pair (trit 2c - 1, trit 2c+1 - 1): shift by 2c, mask the low two
    bits of each half into fp16 1024, subtract 1025.  All 243 x 27 byte pairs, both rows of a
    lane (the second row's bytes one byte higher)."""
    q24, tail = np.meshgrid(np.arange(243), np.arange(27), indexing="ij")
    q24, tail = q24.ravel(), tail.ravel()
    trits = [(q24 // 3 ** j) % 3 for j in range(5)] + [(tail // 3 ** j) % 3 for j in range(3)]
    even = sum(trits[2 * i] << (2 * i) for i in range(4)).astype(np.uint32)
    odd = sum(trits[2 * i + 1] << (2 * i) for i in range(4)).astype(np.uint32)
    for hi in range(2):
        # bytes of the lane's word: (even r, even r+8, odd r, odd r+8); this row's pair at byte hi
        other = (even * 7 + 3) & 0xFF  # some other row's bytes in the neighbouring slots
        word = np.where(hi == 0, even | (other << 8) | (odd << 16) | (other << 24),
                        other | (even << 8) | (other << 16) | (odd << 24)).astype(np.uint64)
        for c in range(4):
            f = ((word >> (2 * c + 8 * hi)) & 0x00030003) | 0x64006400
            lo = bits_to_f64(f & 0xFFFF) - 1025.0
            hi_half = bits_to_f64((f >> 16) & 0xFFFF) - 1025.0
            np.testing.assert_array_equal(lo, trits[2 * c] - 1)
            np.testing.assert_array_equal(hi_half, trits[2 * c + 1] - 1)
