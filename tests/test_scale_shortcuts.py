"""The MS-EDEN pass-1 kernel's shortcut for its pseudo-scale, checked on the
CPU against the oracle's definition E8M3(fp32(g / 6)) (the Quartet II page's
post hoc range alignment: the group maximum over the clip factor, rounded to
an E8M3 pseudo-scale).

The kernel multiplies g by fp32(1/6) instead of dividing: that product lies
within 1.5 ulp of g / 6, hence within one ulp of the correctly rounded
quotient, so the two round to the same E8M3 value unless the product's low
20 mantissa bits lie within two of the rounding midpoint 0x80000; then it
divides exactly.  The GPU self-test (fp4_selftest_arith, counter 5) checks
the kernel over every non-negative fp32 value; this test checks the argument
itself on a strided sample of all non-negative fp32 bit patterns and on
values placed next to every rounding midpoint of several binades."""
import numpy as np

from oracle import formats as fm

F32 = np.float32
U32 = np.uint32


def _e8m3_bits(b):
    """E8M3 round-to-nearest-even of fp32 bit patterns (3 mantissa bits)."""
    b = b.astype(np.uint64)
    r = (b + 0x7FFFF + ((b >> 20) & 1)) & 0xFFF00000
    return r.astype(U32)


def _shortcut(g):
    c = (F32(1.0) / F32(6.0)).astype(F32)
    q = (g * c).astype(F32)
    qb = q.view(U32)
    near = ((qb.astype(np.uint64) + 2 - 0x80000) & 0xFFFFF) <= 4
    exact = (g / F32(6.0)).astype(F32).view(U32)
    return np.where(near, _e8m3_bits(exact), _e8m3_bits(qb)), near


def _definition(g):
    return _e8m3_bits((g / F32(6.0)).astype(F32).view(U32))


def test_reciprocal_of_six():
    c = (F32(1.0) / F32(6.0)).astype(F32)
    assert c.view(U32) == 0x3E2AAAAB
    rel = abs(float(c) - 1.0 / 6.0) * 6.0
    assert rel < 2.0 ** -24                     # |fp32(1/6) - 1/6| / (1/6) below 2^-24


def test_e8m3_bits_matches_the_oracle_rounding():
    rng = np.random.default_rng(3)
    t = rng.uniform(0.0, 1.0, 20000).astype(F32) * np.exp2(rng.integers(-100, 100, 20000)).astype(F32)
    want = fm.e8m3_round(t).view(U32)
    np.testing.assert_array_equal(_e8m3_bits(t.view(U32)), want)


def test_shortcut_on_a_strided_sample_of_all_values():
    with np.errstate(over="ignore"):
        for start in range(0, 0x7F800001, 1 << 27):
            b = np.arange(start, min(start + (1 << 27), 0x7F800001), 61, dtype=np.uint64).astype(U32)
            g = b.view(F32)
            got, _ = _shortcut(g)
            np.testing.assert_array_equal(got, _definition(g))


def test_shortcut_next_to_every_rounding_midpoint():
    """g = 6 x (an E8M3 midpoint) moved by up to 64 ulps either way, in
    binades from the sub-normal range to near the overflow threshold: the
    guard must catch every case where product and quotient round apart."""
    mids = []
    for e in (-140, -126, -100, -20, -1, 0, 1, 7, 20, 100, 124):
        for m in range(8):
            mids.append(np.ldexp(1.0 + (2 * m + 1) / 16.0, e))   # (1 + (m + 1/2) / 8) 2^e
    g0 = (np.array(mids) * 6.0).astype(F32).view(U32).astype(np.int64)
    g = (g0[:, None] + np.arange(-64, 65)[None, :]).reshape(-1)
    g = g[(g > 0) & (g < 0x7F800000)].astype(U32).view(F32)
    got, near = _shortcut(g)
    np.testing.assert_array_equal(got, _definition(g))
    assert near.any()                            # the exact path is exercised
