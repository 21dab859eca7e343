"""The identities the quantiser uses to fold the col transform's 1/4 into the block
maxima and encode multipliers, checked on the CPU in FP32.

Every input is a BF16 value, so every rounded butterfly sum u is a multiple of 2^-133
and u / 4 is exact in FP32 (subnormal or not).  Hence the transform of the 12B NVFP4
page's recipe (the oracle's rht16, which applies the 1/4 last) equals u / 4 exactly,
its block maximum is max|u| / 4, and fl(fl(u / 4) r) = fl(u fl(r / 4)) for every encode
multiplier r >= 2^-124, which covers every tensor scale S <= 2^100."""

import numpy as np

from oracle import nvfp4_oracle as O

F32 = np.float32


def bf16_groups(n, seed):
    """n groups of 16 BF16 values whose exponents span -133 .. 119 (subnormals included),
    mixed signs, so that sums neither overflow nor stay on one scale."""
    rng = np.random.default_rng(seed)
    mant = rng.uniform(1.0, 2.0, (n, 16))
    expo = rng.integers(-133, 120, (n, 1)) + rng.integers(-12, 13, (n, 16))
    x = np.ldexp(mant, np.clip(expo, -140, 120)) * rng.choice([-1.0, 1.0], (n, 16))
    return O.bf16_round(x.astype(F32))


def butterflies(x, signs):
    """The transform's sign flips and stages h = 1, 2, 4, 8 in FP32, without the 1/4."""
    v = np.array(x, dtype=F32, copy=True)
    flip = np.array([(signs >> j) & 1 for j in range(16)], dtype=bool)
    v[..., flip] = -v[..., flip]
    for h in (1, 2, 4, 8):
        for i in range(16):
            if not i & h:
                a, b = v[..., i].copy(), v[..., i + h].copy()
                v[..., i], v[..., i + h] = (a + b).astype(F32), (a - b).astype(F32)
    return v


def test_quarter_of_the_butterflies_is_exact():
    for seed, signs in ((1, 0x5A3C), (2, 0xA53C), (3, 0x0000)):
        x = bf16_groups(20000, seed)
        u = butterflies(x, signs)
        t = O.rht16(x, signs)
        assert np.array_equal(t.astype(np.float64) * 4.0, u.astype(np.float64))      # fl(u / 4) = u / 4
        assert np.array_equal(np.abs(t).max(axis=1), (np.abs(u).max(axis=1) * F32(0.25)).astype(F32))
        assert (np.abs(t)[np.abs(t) > 0] < np.finfo(F32).tiny).any()                 # subnormal results occur


def test_multiplier_fold_matches_two_step_encode():
    x = bf16_groups(4000, 7)
    u = butterflies(x, 0x5A3C)
    t = O.rht16(x, 0x5A3C)
    rng = np.random.default_rng(8)
    # encode multipliers r = fl(1 / fl(s S)) over E4M3 scale bytes and tensor scales up to 2^100
    for log2_s in rng.uniform(-100.0, 100.0, 24):
        S = F32(np.exp2(log2_s))
        for sbyte in rng.integers(1, 127, 6):
            d = F32(O.e4m3_decode(np.array([sbyte], dtype=np.uint8))[0] * S)
            r = F32(F32(1.0) / d)
            if not np.isfinite(r) or r == 0:
                continue
            assert r >= F32(2.0 ** -124)
            with np.errstate(over="ignore"):                   # both sides overflow alike
                two_step = (t * r).astype(F32)
                folded = (u * F32(r * F32(0.25))).astype(F32)
            assert np.array_equal(two_step, folded), (float(S), int(sbyte))


def test_quarter_of_a_tiny_multiplier_can_round():
    """Below 2^-124, r / 4 falls into FP32's subnormal range and may round, which is why
    the kernels fold only while S <= 2^100 (r >= 1 / (448 S) stays far above 2^-124)."""
    r = np.nextafter(F32(2.0 ** -125), F32(1.0))        # 2^-125 + 2^-148
    assert F32(F32(r * F32(0.25)) * F32(4.0)) != r       # r / 4 = 2^-127 + 2^-150 rounds
