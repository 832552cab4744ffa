"""Arithmetic facts the stored-form kernels rely on, checked on the host
against exact integer and rational arithmetic (no GPU):

- the group index of column k as a reciprocal multiply,
  floor((k / 128) / (g / 128)) = ((k >> 7) * ceil(2^16 / (g / 128))) >> 16,
  for every k < 32768 and every group g = 128 q, q <= 256;
- the code-to-float conversion through the exponent field,
  bits(0x4B000000 | c) - 2^23 = c for c < 2^23;
- the product of two fp16 numbers is exact in fp32;
- s c - s z formed from those exact products and rounded once equals the
  exact s (c - z) rounded once to fp32 (what one fused multiply-add gives);
- the 4-bit product's fp16 conversion constants give exact codes from either
  nibble, and its power-of-two scaling of bf16 x into fp16 is exact over the
  range it claims.
"""
from fractions import Fraction

import numpy as np


def test_group_index_reciprocal_is_exact():
    n = np.arange(256, dtype=np.int64)[:, None]            # k >> 7 for k < 32768
    q = np.arange(1, 257, dtype=np.int64)[None, :]         # group / 128
    inv = -(-65536 // q)                                    # ceil(2^16 / q)
    assert np.array_equal((n * inv) >> 16, n // q)


def test_exponent_field_conversion_is_exact():
    c = np.arange(0, 1 << 12, dtype=np.uint32)              # codes (8-bit and well beyond)
    f = (np.uint32(0x4B000000) | c).view(np.float32) - np.float32(8388608.0)
    assert np.array_equal(f, c.astype(np.float32))


def _fp16_sample(rng, n, lo, hi):
    return rng.uniform(lo, hi, n).astype(np.float16)


def test_fp16_products_are_exact_in_fp32():
    rng = np.random.default_rng(0)
    s = np.concatenate([_fp16_sample(rng, 4000, 1e-6, 1.0), np.array([6.1e-5, 65504.0], np.float16)])
    z = np.concatenate([_fp16_sample(rng, 4000, -300.0, 300.0), np.array([-2048.0, 2048.0], np.float16)])
    p32 = s.astype(np.float32) * z.astype(np.float32)
    exact = [Fraction(float(a)) * Fraction(float(b)) for a, b in zip(s, z)]
    assert all(Fraction(float(p)) == e for p, e in zip(p32, exact))


def test_one_rounding_of_the_dequantized_value():
    rng = np.random.default_rng(1)
    n = 20000
    s = _fp16_sample(rng, n, 1e-5, 0.05)
    z = _fp16_sample(rng, n, -8.0, 24.0)                     # off the integers: rounding happens
    c = rng.integers(0, 256, n).astype(np.float32)
    s32, z32 = s.astype(np.float32), z.astype(np.float32)
    # both products are exact in fp32, so one fp32 subtraction rounds the exact difference once
    got = s32 * c - s32 * z32
    rounded = 0
    for i in range(n):
        exact = Fraction(float(s[i])) * (Fraction(int(c[i])) - Fraction(float(z[i])))
        want = np.float32(float(exact))                        # fp64 holds it exactly; one rounding to fp32
        assert Fraction(float(np.float64(float(exact)))) == exact
        assert got[i] == want, (i, float(s[i]), float(z[i]), int(c[i]))
        rounded += Fraction(float(want)) != exact
    assert rounded > 0                                         # the check has teeth: some values do round


def test_fp16_code_conversion_constants():
    """The 4-bit product's conversion: a code c in the low nibble of a half
    ORed into 0x6400 is 1024 + c, and adding 0xE400 (-1024) gives c; in the
    high nibble it is 1024 + 16 c, and times 0x2C00 (1/16) plus 0xD400 (-64)
    gives c.  Every intermediate is exact in fp16."""
    h = lambda bits: np.array([bits], dtype=np.uint16).view(np.float16)[0]  # noqa: E731
    k_sub, k_s16, k_sub64 = h(0xE400), h(0x2C00), h(0xD400)
    assert (float(k_sub), float(k_s16), float(k_sub64)) == (-1024.0, 1.0 / 16, -64.0)
    for c in range(16):
        lo = h(0x6400 | c)
        hi = h(0x6400 | (c << 4))
        assert float(lo) == 1024 + c and float(np.float16(lo + k_sub)) == c
        assert float(hi) == 1024 + 16 * c
        t = np.float16(hi * k_s16)                          # 64 + c, exact
        assert float(t) == 64 + c and float(np.float16(t + k_sub64)) == c


def test_scaled_bf16_values_are_exact_in_fp16():
    """The product scales each 128-column block of bf16 x by a power of two
    that puts its largest magnitude in [2^14, 2^15): every bf16 value from
    2^-28 of that maximum up to it then lies in fp16's normal range
    [2^-14, 2^15], where fp16's 11-bit significand holds bf16's 8 bits."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)                        # every bf16 value
    a = np.abs(v)
    sel = np.isfinite(v) & (a >= 2.0 ** -14) & (a < 2.0 ** 15)
    assert np.array_equal(v[sel].astype(np.float16).astype(np.float32), v[sel])
    assert 2.0 ** 14 * 2.0 ** -28 == 2.0 ** -14               # the range's floor for a block max of 2^14
