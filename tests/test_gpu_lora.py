"""GPU parity of the LoRA-SVD linear against the oracle.

- W_res = BF16(W - L R): bit for bit (FP32 accumulation in a fixed order on both sides).
- U = BF16(A B^T) and Y <- BF16(Y + U C^T): tensor-core products with FP32
  accumulation, held to the GEMM bound of the exact product plus one BF16 half-ulp
  (the BF16 reading), for every rank, both operand layouts, several CTAs and tiles.
- U' = BF16(A B^T / g) (the projection pre-divided by the tensor-scale product g) and
  the NVFP4 GEMM with the rank-r term in its accumulator, BF16(g (A B^T + U V^T)):
  within the GEMM bound over both products plus one BF16 half-ulp, several ranks,
  tiles, a ragged N and a half-empty last row block.
- The composed fprop and dgrad: within that bound plus one BF16 ulp of each U' (each
  side rounds U' on its own), plus the page's claim that the decomposition lowers the
  output error.
- At the 12B up-projection size, sampled rows of every step.
"""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import bf16_to_np

pytestmark = pytest.mark.gpu

SIGNS = 0x5A3C


def bits(x: torch.Tensor) -> np.ndarray:
    return x.view(torch.int16).cpu().numpy().astype(np.uint16)


def to_dev(v: np.ndarray) -> torch.Tensor:
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).cuda()


def svd_factors(w: np.ndarray, rank: int):
    u, s, vt = np.linalg.svd(w.astype(np.float64), full_matrices=False)
    l = O.bf16_round((u[:, :rank] * np.sqrt(s[:rank])).astype(np.float32))
    r = O.bf16_round((np.sqrt(s[:rank])[:, None] * vt[:rank]).astype(np.float32))
    return l, r


def within(got: np.ndarray, pre: np.ndarray, abs_sum: np.ndarray, what: str):
    """The BF16 reading: |got - pre| <= 1e-5 sum|ab| + 1e-6 + 2^-8 |pre|."""
    bound = 1e-5 * abs_sum + 1e-6 + 2.0 ** -8 * np.abs(pre)
    ratio = np.abs(got.astype(np.float64) - pre) / bound
    assert (ratio <= 1.0).all(), "%s: worst ratio %.3g" % (what, float(ratio.max()))


@pytest.mark.parametrize("n,k,rank", [(256, 512, 32), (384, 640, 16), (128, 2048 + 64, 64)])
def test_residual_bit_exact(n, k, rank):
    w = synthetic.normal((n, k), 0.02, seed=n + k, device="cuda")
    wv = bf16_to_np(w)
    l, r = svd_factors(wv, rank)
    got = api.lora_residual(w, to_dev(l), to_dev(r))
    assert (bits(got) == O.f32_to_bf16_bits(O.lora_residual(wv, l, r))).all()
    # factors that do not come from W: larger cancellations
    rng = np.random.default_rng(rank)
    l2 = O.bf16_round(rng.standard_normal((n, rank)).astype(np.float32))
    r2 = O.bf16_round((0.1 * rng.standard_normal((rank, k))).astype(np.float32))
    got = api.lora_residual(w, to_dev(l2), to_dev(r2))
    assert (bits(got) == O.f32_to_bf16_bits(O.lora_residual(wv, l2, r2))).all()


@pytest.mark.parametrize("rank", [16, 32, 48, 64])
@pytest.mark.parametrize("b_trans", [False, True])
def test_project_within_bound(rank, b_trans):
    m, k = 192, 320                                           # 3 CTAs, 5 K-chunks
    a = synthetic.normal((m, k), 1.0, seed=rank, device="cuda", outlier_frac=0.01, outlier_mult=30.0)
    b = synthetic.normal((rank, k), 0.05, seed=rank + 1, device="cuda")
    av, bv = bf16_to_np(a), bf16_to_np(b)
    arg = b.t().contiguous() if b_trans else b
    u = api.lowrank_project(a, arg, b_trans=b_trans)
    within(bf16_to_np(u), O.gemm_ref(av, bv), O.gemm_abs_ref(av, bv), "U")


@pytest.mark.parametrize("m,k,rank", [(208, 320, 16), (208, 320, 48), (19200, 128, 32), (19200, 192, 64)])
@pytest.mark.parametrize("b_trans", [False, True])
def test_project_unit_split(m, k, rank, b_trans):
    """The projection splits M into 16-row units over a persistent grid: 13 units (fewer
    than the SMs, one or none per CTA) and 1200 units (more than eight per CTA on a
    148-SM part, so CTAs take two groups in turn)."""
    a = synthetic.normal((m, k), 1.0, seed=m + rank, device="cuda")
    b = synthetic.normal((rank, k), 0.05, seed=k + rank, device="cuda")
    av, bv = bf16_to_np(a), bf16_to_np(b)
    arg = b.t().contiguous() if b_trans else b
    u = api.lowrank_project(a, arg, b_trans=b_trans)
    within(bf16_to_np(u), O.gemm_ref(av, bv), O.gemm_abs_ref(av, bv), "U")


@pytest.mark.parametrize("rank", [16, 32, 48, 64])
@pytest.mark.parametrize("c_trans", [False, True])
def test_expand_add_within_bound(rank, c_trans):
    m, n = 256, 384                                           # 2 x 3 tiles
    rng = np.random.default_rng(100 + rank)
    y = O.bf16_round(rng.standard_normal((m, n)).astype(np.float32))
    u = O.bf16_round(rng.standard_normal((m, rank)).astype(np.float32))
    c = O.bf16_round((0.1 * rng.standard_normal((n, rank))).astype(np.float32))
    yd = to_dev(y)
    cd = to_dev(c.T.copy()) if c_trans else to_dev(c)
    api.lowrank_expand_add(yd, to_dev(u), cd, c_trans=c_trans)
    pre = y.astype(np.float64) + O.gemm_ref(u, c)
    within(bf16_to_np(yd), pre, O.gemm_abs_ref(u, c), "Y + U C^T")


def lora_bound(parts, c_like, y_ref):
    """|Y_gpu - Y_ref| for the fused LoRA-SVD output: the GEMM bound over both products
    (1e-5 sum|ab| + 1e-6), one BF16 ulp of each U' (2^-7 g |U'| |C|), and one BF16
    half-ulp of the output (2^-8 |Y_ref|)."""
    ul = float(parts["g"]) * (np.abs(parts["u"]).astype(np.float64) @ np.abs(c_like).astype(np.float64).T)
    return 1e-5 * parts["abs_scale"] + 1e-6 + 2.0 ** -7 * ul + 2.0 ** -8 * np.abs(y_ref)


@pytest.mark.parametrize("rank", [16, 32, 48, 64])
@pytest.mark.parametrize("b_trans", [False, True])
def test_project_scaled_within_bound(rank, b_trans):
    m, k = 192, 320
    a = synthetic.normal((m, k), 1.0, seed=rank + 7, device="cuda")
    b = synthetic.normal((rank, k), 0.05, seed=rank + 8, device="cuda")
    sa = torch.tensor([3.0e-3], device="cuda")
    sb = torch.tensor([5.5e-5], device="cuda")
    av, bv = bf16_to_np(a), bf16_to_np(b)
    arg = b.t().contiguous() if b_trans else b
    u = api.lowrank_project_scaled(a, arg, sa, sb, b_trans=b_trans)
    g = np.float32(np.float32(3.0e-3) * np.float32(5.5e-5))
    inv = np.float32(np.float32(1.0) / g)
    # the sum's FP32 rounding may differ from the exact one; then the scaled value is
    # within the GEMM bound of fl32(exact) * inv, and BF16 rounding adds a half-ulp
    pre = O.gemm_ref(av, bv) * float(inv)
    within(bf16_to_np(u), pre, O.gemm_abs_ref(av, bv) * float(inv), "U'")
    exact_path = O.lora_project_scaled(av, bv, g)
    assert np.mean(bf16_to_np(u) == exact_path) > 0.95


@pytest.mark.parametrize("m,n,k,rank", [(256, 256, 256, 32), (384, 640, 512, 16), (512, 384, 1024 + 64, 64),
                                        (768, 512, 768, 48)])
def test_gemm_lowrank_within_bound(m, n, k, rank):
    a = synthetic.normal((m, k), 1.0, seed=m + 1, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
    b = synthetic.normal((n, k), 0.02, seed=n + 2, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    ra, rb = O.quantize(bf16_to_np(a))["row"], O.quantize(bf16_to_np(b))["row"]
    ah, bh = O.dequantize(*ra), O.dequantize(*rb)
    g = np.float32(np.float32(ra[2]) * np.float32(rb[2]))
    rng = np.random.default_rng(rank)
    # U of magnitude 1/g, so that g U V^T is as large as the NVFP4 product
    uv = O.bf16_round((rng.standard_normal((m, rank)) / float(g)).astype(np.float32))
    vv = O.bf16_round((0.3 * rng.standard_normal((n, rank))).astype(np.float32))
    c = api.gemm_lowrank(qa, qb, to_dev(uv), to_dev(vv))
    api.get_status()
    ref = O.gemm_ref(ah, bh) + float(g) * O.gemm_ref(uv, vv)
    scale = O.gemm_abs_ref(ah, bh) + float(g) * O.gemm_abs_ref(uv, vv)
    bound = 1e-5 * scale + 1e-6 + 2.0 ** -8 * np.abs(ref)
    ratio = np.abs(bf16_to_np(c).astype(np.float64) - ref) / bound
    assert (ratio <= 1.0).all(), float(ratio.max())
    # the low-rank term is really there: the plain GEMM misses the reference by far
    plain = bf16_to_np(api.gemm(qa, qb)).astype(np.float64)
    assert (np.abs(plain - ref) / bound).max() > 100


def spiked_weight(n, k, seed):
    rng = np.random.default_rng(seed)
    spike = (rng.standard_normal((n, 4)) @ rng.standard_normal((4, k))) * 0.05
    return O.bf16_round((spike + 0.002 * rng.standard_normal((n, k))).astype(np.float32))


@pytest.mark.parametrize("m,n,k,rank", [(256, 256, 384, 32), (384, 512, 256, 16)])
def test_lora_fwd_and_dgrad(m, n, k, rank):
    wv = spiked_weight(n, k, seed=m + n)
    l, r = svd_factors(wv, rank)
    w_res = O.lora_residual(wv, l, r)
    wq = O.quantize_weight(w_res)
    ld, rd = to_dev(l), to_dev(r)
    w_res_d = api.lora_residual(to_dev(wv), ld, rd)
    assert (bits(w_res_d) == O.f32_to_bf16_bits(w_res)).all()
    wq_row, wq_col = api.quantize_weight(w_res_d)

    x = synthetic.normal((m, k), 1.0, seed=m, device="cuda")
    xv = bf16_to_np(x)
    y, _, _ = api.lora_linear_fwd(x, wq_row, ld, rd, rht_signs=SIGNS)
    y_ref, p = O.lora_linear_fwd(xv, wq, l, r, rht_signs=SIGNS)
    bound = lora_bound(p, l, y_ref)
    err = np.abs(bf16_to_np(y).astype(np.float64) - y_ref)
    assert (err <= bound).all(), float((err / bound).max())
    exact = xv.astype(np.float64) @ wv.T.astype(np.float64)
    y_plain, _, _ = api.linear_fwd(x, api.quantize_weight(to_dev(wv))[0], rht_signs=SIGNS)
    e_lora = np.linalg.norm(bf16_to_np(y) - exact) / np.linalg.norm(exact)
    e_plain = np.linalg.norm(bf16_to_np(y_plain) - exact) / np.linalg.norm(exact)
    assert e_lora < 0.5 * e_plain, (e_lora, e_plain)

    dy = synthetic.normal((m, n), 1e-3, seed=m + 1, device="cuda")
    dyv = bf16_to_np(dy)
    dx, _, _ = api.lora_linear_dgrad(dy, wq_col, ld, to_dev(r.T.copy()), seed=77, offset=3, rht_signs=SIGNS)
    dx_ref, p = O.lora_linear_dgrad(dyv, wq, l, r, seed=77, offset=3, rht_signs=SIGNS)
    bound = lora_bound(p, r.T, dx_ref)
    err = np.abs(bf16_to_np(dx).astype(np.float64) - dx_ref)
    assert (err <= bound).all(), float((err / bound).max())
    api.get_status()


def test_full_size_sampled_rows():
    """The 12B up-projection: W [20480 x 5120], X [16384 x 5120], rank 32.  Rows are
    independent in every step, so sampled rows are checked against the oracle."""
    n, k, m, rank = 20480, 5120, 16384, 32
    w = synthetic.normal((n, k), 0.014, seed=10, device="cuda")
    rng = np.random.default_rng(3)
    l = O.bf16_round((0.05 * rng.standard_normal((n, rank))).astype(np.float32))
    r = O.bf16_round((0.05 * rng.standard_normal((rank, k))).astype(np.float32))
    ld, rd = to_dev(l), to_dev(r)
    w_res = api.lora_residual(w, ld, rd)
    rows = np.sort(rng.choice(n, 48, replace=False))
    want = O.lora_residual(bf16_to_np(w[torch.as_tensor(rows).cuda()]), l[rows], r)
    assert (bits(w_res[torch.as_tensor(rows).cuda()]) == O.f32_to_bf16_bits(want)).all()

    x = synthetic.normal((m, k), 1.0, seed=12, device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    u = api.lowrank_project(x, rd)
    xs = rng.choice(m, 64, replace=False)
    xv = bf16_to_np(x[torch.as_tensor(xs).cuda()])
    within(bf16_to_np(u[torch.as_tensor(xs).cuda()]), O.gemm_ref(xv, r), O.gemm_abs_ref(xv, r), "U rows")

    y = synthetic.normal((m, n), 1.0, seed=13, device="cuda")
    u_in = synthetic.normal((m, rank), 1.0, seed=14, device="cuda")         # an input of its own, not U above
    y0 = bf16_to_np(y[torch.as_tensor(xs).cuda()])
    uv = bf16_to_np(u_in[torch.as_tensor(xs).cuda()])
    api.lowrank_expand_add(y, u_in, ld)
    pre = y0.astype(np.float64) + O.gemm_ref(uv, l)
    within(bf16_to_np(y[torch.as_tensor(xs).cuda()]), pre, O.gemm_abs_ref(uv, l), "Y rows")
    api.get_status()
