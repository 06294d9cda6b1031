"""CPU check of the threshold form of the 2-bit code used by the quantizer kernel.

With a stored fp16 scale s > 0 and d = fl(x - z), the definition
clamp(rint(fl(d / s)), 0, 3) (IEEE fp32 division, rint half to even) equals
[d > s/2] + [d > pred(1.5 s)] + [d > 2.5 s], because division and rounding are
monotone and s has at most 11 significant bits, so s/2, 1.5 s and 2.5 s are
exact in fp32 and each rounding boundary times s falls inside one fp32 ulp
beside them.  This replays both forms in numpy float32 on quotients at, and a
few ulps around, every boundary and everywhere else, for normal and subnormal
fp16 scales, and requires them to agree; an unshifted middle bound (1.5 s) or a
>= on the outer bounds fails it.
"""
import numpy as np


def fp16_scales(rng, n):
    bits = rng.integers(1, 0x7BFF, n, dtype=np.uint16)
    return bits.view(np.float16).astype(np.float32)


def threshold_codes(d, s, e2):
    e1 = (s * np.float32(0.5)).astype(np.float32)
    e3 = (s * np.float32(2.5)).astype(np.float32)
    return (d > e1).astype(np.int32) + (d > e2).astype(np.int32) + (d > e3).astype(np.int32)


def defined_codes(d, s):
    return np.clip(np.rint((d / s).astype(np.float32)), 0, 3).astype(np.int32)


def cases(seed, n=600_000):
    rng = np.random.default_rng(seed)
    s = fp16_scales(rng, n)
    which = rng.integers(0, 4, n)
    base = np.choose(which, [s * np.float32(0.5), s * np.float32(1.5), s * np.float32(2.5),
                             s * np.float32(1.0)]).astype(np.float32)
    step = rng.integers(-6, 7, n).astype(np.int32)
    near = (base.view(np.int32) + step).view(np.float32)
    spread = (rng.uniform(-0.5, 3.5, n) * s).astype(np.float32)
    d = np.where(rng.random(n) < 0.75, near, spread).astype(np.float32)
    return d, s


def test_threshold_form_equals_definition():
    for seed in range(3):
        d, s = cases(seed)
        e2 = np.nextafter((s * np.float32(1.5)).astype(np.float32), np.float32(-np.inf))
        assert np.array_equal(threshold_codes(d, s, e2), defined_codes(d, s))


def test_plausible_mistakes_are_caught():
    d, s = cases(7)
    ref = defined_codes(d, s)
    # the middle bound without its one-ulp shift: ties at 1.5 round to 2
    e2_wrong = (s * np.float32(1.5)).astype(np.float32)
    assert not np.array_equal(threshold_codes(d, s, e2_wrong), ref)
    # >= on the outer bounds: ties at 0.5 and 2.5 round down (to even)
    e1 = (s * np.float32(0.5)).astype(np.float32)
    e2 = np.nextafter((s * np.float32(1.5)).astype(np.float32), np.float32(-np.inf))
    e3 = (s * np.float32(2.5)).astype(np.float32)
    ge = (d >= e1).astype(np.int32) + (d > e2).astype(np.int32) + (d >= e3).astype(np.int32)
    assert not np.array_equal(ge, ref)
