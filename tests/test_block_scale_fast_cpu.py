"""The quantiser's one-multiply block scale, checked on the CPU in FP32.

The block scale of the 12B NVFP4 page's format is s = E4M3(fl(fl(b / 6) / S)) (the
oracle's definition).  For 1D blocks the kernels compute s_a = fl(b K) with
K = fl(1 / fl(6 S)) (K = 0 for S < 2^-100) and keep it when s_a >= 2^-6 and the 20
FP32 mantissa bits below E4M3's three lie more than 16 away from 0x80000 (the midpoint
between two E4M3 values); otherwise they do the two divisions.  s_a and the exact scale
are within 5 FP32 ulps of each other, so wherever s_a is kept both give the same E4M3
byte.  These tests check that on random and on adversarial (near-midpoint) inputs, and
that the near-midpoint cases do reach the division path."""

import numpy as np

from oracle import nvfp4_oracle as O

F32 = np.float32


def fast_factor(S):
    S = np.asarray(S, dtype=F32)
    with np.errstate(divide="ignore", over="ignore"):
        K = (F32(1.0) / (F32(6.0) * S).astype(F32)).astype(F32)
    return np.where((S >= F32(2.0 ** -100)) & np.isfinite(K), K, F32(0.0)).astype(F32)


def kept(b, K):
    """The kernels' acceptance test for s_a = fl(b K)."""
    with np.errstate(over="ignore", invalid="ignore"):
        sa = (np.asarray(b, dtype=F32) * K).astype(F32)
    dm = (sa.view(np.uint32) & np.uint32(0xFFFFF)).astype(np.int64) - 0x80000
    return sa, (sa >= F32(2.0 ** -6)) & (np.abs(dm) > 16)


def exact_scale(b, S):
    with np.errstate(over="ignore"):
        return ((np.asarray(b, dtype=F32) / F32(6.0)).astype(F32) / np.asarray(S, dtype=F32)).astype(F32)


def check(b, S):
    K = fast_factor(S)
    sa, ok = kept(b, K)
    s = exact_scale(b, S)
    use = ok & np.isfinite(s) & np.isfinite(sa)
    assert np.array_equal(O.e4m3_encode(sa[use]), O.e4m3_encode(s[use]))
    return ok


def test_random_blocks_and_tensor_scales():
    rng = np.random.default_rng(11)
    n = 400000
    b = np.ldexp(rng.uniform(1.0, 2.0, n), rng.integers(-130, 127, n)).astype(F32)
    S = np.ldexp(rng.uniform(1.0, 2.0, n), rng.integers(-110, 120, n)).astype(F32)
    ok = check(b, S)
    assert ok.mean() > 0.2                      # the fast path is the common case


def test_blocks_next_to_e4m3_midpoints():
    """b set so that the exact scale lands within 40 FP32 ulps of a rounding midpoint
    of E4M3 (normal range), for tensor scales from 2^-100 to 2^100."""
    rng = np.random.default_rng(12)
    mids = np.array([(1.0 + (2 * k + 1) / 16.0) * 2.0 ** e for e in range(-6, 9) for k in range(8)
                     if (1.0 + (2 * k + 1) / 16.0) * 2.0 ** e < 448.0])
    S = np.ldexp(rng.uniform(1.0, 2.0, 64), rng.integers(-100, 101, 64)).astype(F32)
    rejected = 0
    for Si in S:
        m = F32(mids[rng.integers(0, len(mids), 400)])
        target = (m * F32(6.0)).astype(F32) * Si                     # b ~ 6 S m
        base = target.astype(F32).view(np.int32).astype(np.int64)
        b = (base + rng.integers(-40, 41, base.shape)).astype(np.int32).view(F32)
        ok = check(b, np.full(b.shape, Si, dtype=F32))
        rejected += int((~ok).sum())
    assert rejected > 0                          # near a midpoint the divisions are taken
