"""The decode kernel's RoPE angle reduction, checked in exact arithmetic.

Pre-RoPE decode rotates keys by angles a = fl32(position * inv_freq) and takes
sin/cos of a - k*2pi, k = rint(a/2pi), computed with four fp32 FMAs against
2pi = P1 + P2 + P3 + P4 (Cody and Waite's method; KIVI article, paragraph 4,
for where RoPE enters).  This emulates that fp32 sequence exactly (each FMA
rounded once, to nearest even) and checks the reduced angle against
a - k*2pi in rational arithmetic, across the positions a pre-RoPE cache may
hold (up to its 823,000-token limit) and the frequencies of theta = 1e4 and
5e5 at head dims 64 and 128.
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest

# 2pi to 100 digits.
TWO_PI = Fraction("6.283185307179586476925286766559005768394338798750211641949889184615632812572417997256069650684234136")
# The kernel's constants, as fp32 bit patterns.
INV_2PI = 0x3E22F983
P = [0x40CA0000, 0xBCF00000, 0xB7960000, 0x338885A3]
MAGIC = Fraction(12582912)


def f32_bits(b):
    return Fraction(struct.unpack(">f", b.to_bytes(4, "big"))[0])


def rne32(x: Fraction) -> Fraction:
    """Round to the nearest fp32 value, ties to even (no overflow here)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = math.floor(math.log2(x.numerator) - math.log2(x.denominator))
    while Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    e = max(e, -126)
    scaled = x * Fraction(2) ** (23 - e)
    q, rem = divmod(scaled.numerator, scaled.denominator)
    twice = 2 * rem
    if twice > scaled.denominator or (twice == scaled.denominator and q % 2 == 1):
        q += 1
    return sign * Fraction(q) * Fraction(2) ** (e - 23)


def reduce_like_kernel(a: Fraction):
    k = rne32(rne32(a * f32_bits(INV_2PI) + MAGIC) - MAGIC)
    r = a
    for b in P:
        r = rne32(-k * f32_bits(b) + r)
    return k, r


def inv_freqs(theta, D):
    return [Fraction(float(np.float32(theta ** (-2.0 * i / D)))) for i in range(D // 2)]


def test_constants_split_two_pi():
    parts = [f32_bits(b) for b in P]
    assert abs(sum(parts) - TWO_PI) < Fraction(1, 2 ** 50)
    # P1..P3 carry at most 7 significant bits, so k*P_i is exact in fp32 for k < 2^17.
    for p in parts[:3]:
        m = abs(p)
        while m.denominator != 1:
            m *= 2
        assert m.numerator.bit_length() - (m.numerator & -m.numerator).bit_length() + 1 <= 7


@pytest.mark.parametrize("theta,D", [(10000.0, 128), (10000.0, 64), (500000.0, 128)])
def test_reduced_angle_within_2_to_minus_22(theta, D):
    rng = np.random.default_rng(3)
    positions = sorted(set([0, 1, 2, 31, 32, 4095, 131071, 131072, 131103, 822999]
                           + rng.integers(0, 823000, 40).tolist()))
    freqs = inv_freqs(theta, D)
    picks = sorted(set([0, 1, 2, len(freqs) - 1] + rng.integers(0, len(freqs), 6).tolist()))
    worst = Fraction(0)
    for pos in positions:
        for i in picks:
            a = rne32(Fraction(pos) * freqs[i])
            k, r = reduce_like_kernel(a)
            exact = a - k * TWO_PI
            err = abs(r - exact)
            worst = max(worst, err)
            assert abs(r) <= Fraction(355, 113) + Fraction(1, 2 ** 20), (pos, i, float(r))
    assert worst <= Fraction(1, 2 ** 22), float(worst)
