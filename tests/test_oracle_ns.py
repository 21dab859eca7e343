"""Pins of the oracle's NVFP4 Newton-Schulz iteration (cubic, residual form) against
what the mathematics fixes: closed forms on signed partial permutations, the
orthogonal fixed point, exact normalisation cases and convergence towards the
orthogonal polar factor that an SVD gives."""

import numpy as np
import pytest

from oracle import nvfp4_oracle as O


def signed_partial_permutation(m, n, seed):
    """[m x n], m <= n: one +-1 per row, in distinct columns (orthonormal rows)."""
    rng = np.random.default_rng(seed)
    p = np.zeros((m, n), dtype=np.float32)
    cols = rng.permutation(n)[:m]
    p[np.arange(m), cols] = rng.choice([-1.0, 1.0], m)
    return p


@pytest.mark.parametrize("m,n", [(32, 64), (48, 48), (16, 128)])
def test_step_closed_form_on_scaled_permutation(m, n):
    """X = c P with c = 21/32 = 2688 * 2^-12: NVFP4 holds c P exactly (tensor scale 2^-12,
    block scale 448, code 6), X X^T = c^2 I exactly, R = BF16(1 - c^2) I = (73/128) I,
    and X' = BF16(c + c * 73/256) P = (27/32) P.  The scalar cubic map 3c/2 - c^3/2 =
    0.8431 rounds to the same BF16 value."""
    c = np.float32(21 / 32)
    p = signed_partial_permutation(m, n, seed=m + n)
    x_new, parts = O.ns_step(c * p)
    assert np.array_equal(parts["x_row"], c * p) and np.array_equal(parts["x_col"], (c * p).T)
    assert np.array_equal(parts["r"], np.float32(73 / 128) * np.eye(m, dtype=np.float32))
    assert np.array_equal(x_new, np.float32(27 / 32) * p)
    scalar_map = 1.5 * (21 / 32) - 0.5 * (21 / 32) ** 3
    assert O.bf16_round(np.float32(scalar_map)) == np.float32(27 / 32)


def test_orthogonal_rows_are_a_fixed_point():
    p = signed_partial_permutation(32, 96, seed=3)
    x_new, _ = O.ns_step(p)
    assert np.array_equal(x_new, p)


def test_zero_is_a_fixed_point():
    x = np.zeros((32, 64), dtype=np.float32)
    x_new, parts = O.ns_step(x)
    assert np.array_equal(x_new, x)
    assert np.array_equal(parts["r"], np.eye(32, dtype=np.float32))
    g, nrm = O.newton_schulz(x, 3)
    assert nrm == 0 and not g.any()


def test_normalize_exact_case_and_scale_invariance():
    """G = +-3 with m n = 4^k: ||G||_F = 3 * 2^k exactly and X_0 = +-2^-k; scaling G by
    a power of two leaves X_0 unchanged."""
    rng = np.random.default_rng(11)
    m, n = 64, 256                              # m n = 2^14 -> ||G|| = 3 * 2^7
    g = (3.0 * rng.choice([-1.0, 1.0], (m, n))).astype(np.float32)
    x0, nrm = O.ns_normalize(g)
    assert nrm == np.float32(384.0)
    assert np.array_equal(np.abs(x0), np.full((m, n), 2.0 ** -7, dtype=np.float32))
    assert np.array_equal(np.sign(x0), np.sign(g))
    g2 = O.bf16_round(rng.standard_normal((m, n)).astype(np.float32))
    a, na = O.ns_normalize(g2)
    b, nb = O.ns_normalize(g2 * np.float32(2.0 ** 5))
    assert np.array_equal(a, b) and nb == na * np.float32(32.0)
    fro = np.sqrt((a.astype(np.float64) ** 2).sum())
    assert abs(fro - 1.0) < 2.0 ** -8                 # BF16 rounding of each element only


def test_frobenius_norm_against_library():
    rng = np.random.default_rng(4)
    g = O.bf16_round(rng.standard_t(3, (128, 96)).astype(np.float32))
    want = np.linalg.norm(g.astype(np.float64))
    assert abs(float(O.frobenius_norm(g)) - want) <= 2.0 ** -23 * want


def test_add_product_rounding_order():
    """C <- BF16(fl32(fl32(P) + C)): P = 2^-8 + 2^-40 rounds to 2^-8 in FP32, so 1 + P
    becomes the exact BF16 tie 1 + 2^-8, which goes to the even 1.0; a single rounding
    of the exact sum would give 1 + 2^-7."""
    got = O.add_product_bf16(np.array([2.0 ** -8 + 2.0 ** -40]), np.array([1.0], dtype=np.float32))
    assert got[0] == np.float32(1.0)
    got = O.add_product_bf16(np.array([2.0 ** -8 + 2.0 ** -20]), np.array([1.0], dtype=np.float32))
    assert got[0] == np.float32(1.0 + 2.0 ** -7)


def test_converges_towards_polar_factor():
    """From G = U diag(sigma) V^T with sigma in [0.2, 1] (condition 5): twelve NVFP4
    steps put every singular value within 15 % of 1 and X near U V^T; the residual form
    keeps the 4-bit error in the correction term, so the spread settles near 10 %."""
    rng = np.random.default_rng(5)
    m, n = 32, 64
    u, _ = np.linalg.qr(rng.standard_normal((m, m)))
    v, _ = np.linalg.qr(rng.standard_normal((n, m)))
    g = O.bf16_round((((u * np.linspace(0.2, 1.0, m)) @ v.T) * 3.0).astype(np.float32))
    uu, _, vt = np.linalg.svd(g.astype(np.float64), full_matrices=False)
    polar = uu @ vt
    x, nrm = O.newton_schulz(g, 12)
    assert abs(float(nrm) - np.linalg.norm(g.astype(np.float64))) < 1e-5 * float(nrm)
    sv = np.linalg.svd(x.astype(np.float64), compute_uv=False)
    assert 0.85 < sv.min() and sv.max() < 1.15, sv
    assert np.linalg.norm(x - polar) / np.sqrt(m) < 0.16
    x0, _ = O.newton_schulz(g, 0)
    assert np.linalg.norm(x0 - polar) / np.sqrt(m) > 0.8                   # far before iterating


def test_spectrum_generator_has_the_requested_singular_values():
    """The seeded Newton-Schulz inputs: U diag(sigma) V^T with orthonormal factors, so the
    singular values are the requested ones up to BF16 rounding of the entries."""
    from nvfp4_pretraining_linear_b200 import synthetic
    g = synthetic.spectrum(64, 160, 0.1, 1.0, seed=3).float().numpy().astype(np.float64)
    sv = np.sort(np.linalg.svd(g, compute_uv=False))
    want = np.linspace(0.1, 1.0, 64)
    assert np.abs(sv - want).max() < 2e-3
    again = synthetic.spectrum(64, 160, 0.1, 1.0, seed=3).float().numpy()
    assert np.array_equal(again, g.astype(np.float32))                      # seeded
