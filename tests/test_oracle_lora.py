"""Pins of the oracle's LoRA-SVD linear (NVFP4 residual weight plus a BF16 low-rank
branch that joins the NVFP4 accumulator): the decomposition is an identity without
quantisation, zero factors reduce it to the plain NVFP4 linear, the residual's FP32
accumulation order is the stated one, the low-rank products (plain and pre-divided by
the tensor-scale product) match brute force, a power-of-two scale product divides out
exactly, and -- the claim of the page -- moving the top singular directions out of the
4-bit path lowers the error of the layer's output."""

import numpy as np
import pytest

from oracle import nvfp4_oracle as O


def small_ints(shape, lo, hi, seed):
    return np.random.default_rng(seed).integers(lo, hi + 1, shape).astype(np.float32)


def test_residual_of_an_exact_low_rank_weight_is_zero():
    l, r = small_ints((64, 16), -2, 2, 1), small_ints((16, 96), -2, 2, 2)
    w = (l.astype(np.float64) @ r.astype(np.float64)).astype(np.float32)      # |w| <= 64: exact in BF16
    assert not O.lora_residual(w, l, r).any()
    assert np.array_equal(O.lora_residual(w, np.zeros_like(l), r), w)


def test_residual_accumulates_in_fp32_in_order():
    """Products 2^24, 1, -2^24 in that order: FP32 gives 2^24 + 1 = 2^24 (tie to even), then
    0, so W_res = W; the exact sum 1 would give W - 1."""
    l = np.array([[4096.0, 1.0, -4096.0]], dtype=np.float32)
    r = np.array([[4096.0], [1.0], [4096.0]], dtype=np.float32)
    w = np.array([[3.0]], dtype=np.float32)
    assert O.lora_residual(w, l, r)[0, 0] == np.float32(3.0)
    l2 = np.array([[1.0, 4096.0, -4096.0]], dtype=np.float32)                    # 1 first: 1 + 2^24 rounds too
    r2 = np.array([[1.0], [4096.0], [4096.0]], dtype=np.float32)
    assert O.lora_residual(w, l2, r2)[0, 0] == np.float32(3.0)
    l3 = np.array([[4096.0, -4096.0, 1.0]], dtype=np.float32)                    # cancellation first: exact
    r3 = np.array([[4096.0], [4096.0], [1.0]], dtype=np.float32)
    assert O.lora_residual(w, l3, r3)[0, 0] == np.float32(2.0)


def test_decomposition_is_an_identity_without_quantisation():
    m, n, k, rank = 32, 48, 64, 16
    x = small_ints((m, k), -1, 1, 3)
    w = small_ints((n, k), -3, 3, 4)
    l, r = small_ints((n, rank), -1, 1, 5), small_ints((rank, k), -1, 1, 6)
    w_res = O.lora_residual(w, l, r)
    assert np.array_equal(w_res, w - (l.astype(np.float64) @ r).astype(np.float32))
    y, parts = O.lora_linear_fwd(x, w_res, l, r, quantize_operands=False)
    assert np.array_equal(y, (x.astype(np.float64) @ w.T.astype(np.float64)).astype(np.float32))
    dy = small_ints((m, n), -1, 1, 7)
    dx, _ = O.lora_linear_dgrad(dy, w_res, l, r, seed=0, offset=0, quantize_operands=False)
    assert np.array_equal(dx, (dy.astype(np.float64) @ w.astype(np.float64)).astype(np.float32))


def test_zero_factors_reduce_to_the_plain_linear():
    rng = np.random.default_rng(8)
    x = O.bf16_round(rng.standard_normal((64, 128)).astype(np.float32))
    w = O.bf16_round((0.02 * rng.standard_normal((96, 128))).astype(np.float32))
    l, r = np.zeros((96, 16), np.float32), O.bf16_round(rng.standard_normal((16, 128)).astype(np.float32))
    wq = O.quantize_weight(O.lora_residual(w, l, r))
    y, parts = O.lora_linear_fwd(x, wq, l, r, rht_signs=0x5A3C)
    y_plain, (ah, bh), _ = O.linear_fwd_ref(x, O.quantize_weight(w), rht_signs=0x5A3C)
    assert np.array_equal(y, y_plain)
    assert np.array_equal(parts["abs_scale"], O.gemm_abs_ref(ah, bh))
    dy = O.bf16_round((1e-3 * rng.standard_normal((64, 96))).astype(np.float32))
    dx, _ = O.lora_linear_dgrad(dy, wq, l, r, seed=5, offset=0, rht_signs=0x5A3C)
    dx_plain, _, _ = O.linear_dgrad_ref(dy, O.quantize_weight(w), 5, 0, rht_signs=0x5A3C)
    assert np.array_equal(dx, dx_plain)


def test_low_rank_products_match_brute_force():
    rng = np.random.default_rng(9)
    a = O.bf16_round(rng.standard_normal((5, 32)).astype(np.float32))
    b = O.bf16_round(rng.standard_normal((4, 32)).astype(np.float32))
    u = O.lora_project(a, b)
    for i in range(5):
        for j in range(4):
            s = sum(float(a[i, k]) * float(b[j, k]) for k in range(32))            # exact enough in binary64
            assert u[i, j] == O.bf16_round(np.float32(s))
    y = O.bf16_round(rng.standard_normal((5, 6)).astype(np.float32))
    c = O.bf16_round(rng.standard_normal((6, 4)).astype(np.float32))
    got = O.lora_expand_add(y, u, c)
    for i in range(5):
        for j in range(6):
            v = np.float32(sum(float(u[i, t]) * float(c[j, t]) for t in range(4)))
            assert got[i, j] == O.bf16_round(np.float32(v + y[i, j]))


def test_moving_top_singular_directions_out_of_fp4_lowers_the_error():
    """W = a rank-4 spike plus small noise.  With L R the top-16 SVD part of W, the
    layer's output error against the exact X W^T falls well below that of plain NVFP4."""
    rng = np.random.default_rng(10)
    m, n, k, rank = 128, 256, 256, 16
    x = O.bf16_round(rng.standard_normal((m, k)).astype(np.float32))
    spike = (rng.standard_normal((n, 4)) @ rng.standard_normal((4, k))) * 0.05
    w = O.bf16_round((spike + 0.002 * rng.standard_normal((n, k))).astype(np.float32))
    u, s, vt = np.linalg.svd(w.astype(np.float64), full_matrices=False)
    l = O.bf16_round((u[:, :rank] * np.sqrt(s[:rank])).astype(np.float32))
    r = O.bf16_round((np.sqrt(s[:rank])[:, None] * vt[:rank]).astype(np.float32))
    exact = x.astype(np.float64) @ w.T.astype(np.float64)
    y_plain, _, _ = O.linear_fwd_ref(x, O.quantize_weight(w))
    y_lora, _ = O.lora_linear_fwd(x, O.quantize_weight(O.lora_residual(w, l, r)), l, r)
    e_plain = np.linalg.norm(y_plain - exact) / np.linalg.norm(exact)
    e_lora = np.linalg.norm(y_lora - exact) / np.linalg.norm(exact)
    assert e_lora < 0.5 * e_plain, (e_lora, e_plain)


def test_scaled_projection_matches_brute_force():
    """U' = BF16(fl32(fl32(sum) * fl32(1 / g))) element by element, for a g that is not a
    power of two; and for g = 2^-9 the division is exact, so U' g equals the plain U."""
    rng = np.random.default_rng(11)
    a = O.bf16_round(rng.standard_normal((6, 48)).astype(np.float32))
    b = O.bf16_round(rng.standard_normal((5, 48)).astype(np.float32))
    g = np.float32(3.0e-4)
    inv = np.float32(np.float32(1.0) / g)
    u = O.lora_project_scaled(a, b, g)
    for i in range(6):
        for j in range(5):
            s = np.float32(sum(float(a[i, k]) * float(b[j, k]) for k in range(48)))
            assert u[i, j] == O.bf16_round(np.float32(s * inv))
    g2 = np.float32(2.0 ** -9)
    assert np.array_equal(O.lora_project_scaled(a, b, g2) * g2, O.lora_project(a, b))


def test_fused_reference_adds_the_scaled_low_rank_product():
    """The fused reference is the NVFP4 product plus g U' L^T, where g is the product of
    the two tensor scales: checked against a hand composition from the quantised layouts
    (a wrong scale, a missing factor g or a transposed factor fails it)."""
    rng = np.random.default_rng(12)
    m, n, k, rank = 32, 64, 96, 16
    x = O.bf16_round(rng.standard_normal((m, k)).astype(np.float32))
    w = O.bf16_round((0.02 * rng.standard_normal((n, k))).astype(np.float32))
    l = O.bf16_round((0.05 * rng.standard_normal((n, rank))).astype(np.float32))
    r = O.bf16_round((0.05 * rng.standard_normal((rank, k))).astype(np.float32))
    wq = O.quantize_weight(O.lora_residual(w, l, r))
    y, parts = O.lora_linear_fwd(x, wq, l, r)
    xq = O.quantize(x, emit_row=True)["row"]
    g = np.float32(np.float32(xq[2]) * np.float32(wq["row"][2]))
    assert parts["g"] == g
    u = O.bf16_round((np.float32(1.0) / g * (x.astype(np.float64) @ r.T.astype(np.float64)).astype(np.float32))
                     .astype(np.float32))
    want = O.dequantize(*xq).astype(np.float64) @ O.dequantize(*wq["row"]).astype(np.float64).T + \
        float(g) * (u.astype(np.float64) @ l.T.astype(np.float64))
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    # g U' approximates the plain projection within one BF16 rounding
    plain = x.astype(np.float64) @ r.T.astype(np.float64)
    assert np.all(np.abs(float(g) * parts["u"] - plain) <= 2.0 ** -8 * np.abs(plain) + 1e-30)
