"""CPU check of the code decision used by the diagnostic quantizer kernel.

The kernel needs rint(RN(d/s)) clamped to [lo, L] (IEEE fp32 division, ties to
even).  It takes q = RN(d * RN(1/s)), rounds clamp(q) to an integer by adding
and subtracting 1.5 * 2^23, and falls back to the IEEE division only when Ziv's
rounding test fails (A. Ziv, "Fast evaluation of elementary mathematical
functions with correctly rounded last bit", ACM TOMS 17(3), 1991): q within
2^-13 of a half-integer while the residual d - q*s is not exactly zero.  This
test replays that decision in numpy float32 arithmetic (IEEE, one rounding per
operation) on millions of quotients, most of them at or next to half-integers,
for every width and both code ranges, and requires it to equal the definition.
"""
import numpy as np
import pytest

ROUND = np.float32(12582912.0)        # 1.5 * 2^23
NEAR = np.float32(0.5 - 2.0 ** -13)


def fp16_scales(rng, n):
    """Positive finite fp16 values (normal and subnormal) as float32."""
    bits = rng.integers(1, 0x7BFF, n, dtype=np.uint16)
    return bits.view(np.float16).astype(np.float32)


def fast_codes(d, s, lo, L):
    rs = (np.float32(1.0) / s).astype(np.float32)
    q = (d * rs).astype(np.float32)
    y = np.minimum(np.maximum(q, lo), L).astype(np.float32)
    r = ((y + ROUND).astype(np.float32) - ROUND).astype(np.float32)
    window = np.abs((y - r).astype(np.float32)) > NEAR
    # residual d - q*s: q*s is exact in float64 and a difference of distinct
    # float64 values is never 0, so this is 0 exactly when q*s == d
    inexact = (d.astype(np.float64) - q.astype(np.float64) * s.astype(np.float64)) != 0.0
    slow = window & inexact
    exact_y = np.minimum(np.maximum((d / s).astype(np.float32), lo), L).astype(np.float32)
    exact_r = ((exact_y + ROUND).astype(np.float32) - ROUND).astype(np.float32)
    return np.where(slow, exact_r, r), slow


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_fast_quotient_equals_ieee_rint(sym, bits):
    if sym and bits < 2:
        pytest.skip("symmetric codes need two bits")
    rng = np.random.default_rng(bits + 10 * sym)
    n = 400_000
    L = np.float32((1 << (bits - 1)) - 1 if sym else (1 << bits) - 1)
    lo = np.float32(-L - 1 if sym else 0.0)
    s = fp16_scales(rng, n)
    k = rng.integers(int(lo) - 1, int(L) + 1, n).astype(np.float32)
    mid = ((k + np.float32(0.5)) * s).astype(np.float32)          # exact products
    kind = rng.integers(0, 3, n)
    step = rng.integers(-4, 5, n).astype(np.int32)
    near = (mid.view(np.int32) + step).view(np.float32)            # a few ulps away
    uniform = (((lo - 1) + rng.random(n) * (L - lo + 2)) * s).astype(np.float32)
    d = np.where(kind == 0, mid, np.where(kind == 1, near, uniform)).astype(np.float32)
    got, slow = fast_codes(d, s, lo, L)
    ref = np.minimum(np.maximum(np.rint((d / s).astype(np.float32)), lo), L)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]
    assert not np.signbit(got[got == 0]).any()
    # spread quotients rarely need the division (the window is 2^-12 wide per
    # half-integer), and the exact-residual filter keeps most exact
    # half-integer quotients (q*s == d) on the fast path
    assert slow[kind == 2].mean() < 1e-3
    assert slow[kind == 0].mean() < 0.2
