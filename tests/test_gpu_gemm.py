"""GPU parity of the block-scaled NVFP4 GEMM (nvfp4_gemm) against the oracle's
FP64 product of the dequantised operands.

Bound: |C - C_ref| <= 1e-5 * sum_k |a_k b_k| + 1e-6 for FP32 output; the BF16
output adds one BF16 half-ulp (2^-8 |C_ref|) for its final rounding."""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import assert_layout_equal, bf16_to_np, gemm_check

pytestmark = pytest.mark.gpu

SHAPES = [
    (128, 128, 64),       # one tile, one MMA k-step
    (256, 256, 256),      # tiny config
    (384, 640, 320),      # N tail of 128 (half tile), K tail of 64
    (512, 384, 1024),
    (256, 1280, 768),     # several N tiles, K tail of 0
    (1152, 512, 2112),    # 10 pair tiles (one wave), half-empty last row block, K tail of 64
    (128, 20480, 320),    # 128 rows and more 256-column tiles than CTA pairs: the single-CTA kernel
]


def random_shapes(n, seed):
    """Seeded shapes over the GEMM's constraints (M, N multiples of 128, K of 64): one
    or several pair tiles, half-empty row blocks (M % 256 == 128), N tails of 128 and
    every K tail (K % 256 in {0, 64, 128, 192})."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        out.append((128 * int(rng.integers(1, 9)), 128 * int(rng.integers(1, 7)), 64 * int(rng.integers(1, 21))))
    return out


def operands(M, N, K, seed, kind="outliers"):
    if kind == "outliers":
        a = synthetic.normal((M, K), 1.0, seed=seed, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
        b = synthetic.normal((N, K), 1.0, seed=seed + 1, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
    else:
        a = synthetic.student_t((M, K), 3, 0.1, seed=seed, device="cuda")
        b = synthetic.normal((N, K), 0.02, seed=seed + 1, device="cuda")
    return a, b


def quantised_pair(a, b):
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    ra = O.quantize(bf16_to_np(a))["row"]
    rb = O.quantize(bf16_to_np(b))["row"]
    assert_layout_equal(qa, ra, "A")
    assert_layout_equal(qb, rb, "B")
    return qa, qb, O.dequantize(*ra), O.dequantize(*rb)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_f32_within_bound(M, N, K):
    a, b = operands(M, N, K, seed=M + N + K)
    qa, qb, ah, bh = quantised_pair(a, b)
    c = api.gemm(qa, qb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ratio = gemm_check(c.cpu().numpy(), ah, bh)
    assert ratio <= 1.0, ratio


@pytest.mark.parametrize("M,N,K", random_shapes(12, 2026))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_random_shapes_within_bound(M, N, K, out_dtype):
    a, b = operands(M, N, K, seed=3 * M + 5 * N + K, kind="t" if out_dtype == torch.bfloat16 else "outliers")
    qa, qb, ah, bh = quantised_pair(a, b)
    c = api.gemm(qa, qb, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ratio = gemm_check(c.float().cpu().numpy(), ah, bh, bf16=out_dtype == torch.bfloat16)
    assert ratio <= 1.0, (M, N, K, ratio)


@pytest.mark.parametrize("M,N,K", SHAPES[:4])
def test_gemm_bf16_within_bound(M, N, K):
    a, b = operands(M, N, K, seed=7 * M + K, kind="t")
    qa, qb, ah, bh = quantised_pair(a, b)
    c = api.gemm(qa, qb, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ratio = gemm_check(c.float().cpu().numpy(), ah, bh, bf16=True)
    assert ratio <= 1.0, ratio


def test_gemm_alpha_and_accumulate():
    M, N, K = 256, 384, 512
    a, b = operands(M, N, K, seed=99)
    qa, qb, ah, bh = quantised_pair(a, b)
    g = torch.Generator(device="cuda").manual_seed(5)
    c0 = torch.randn((M, N), generator=g, device="cuda") * 10
    c = c0.clone()
    api.gemm(qa, qb, alpha=0.375, accumulate=True, out=c)
    torch.cuda.synchronize()
    ratio = gemm_check(c.cpu().numpy(), ah, bh, alpha=0.375, c0=c0.cpu().numpy())
    assert ratio <= 1.0, ratio
    cb0 = c0.to(torch.bfloat16)
    cb = cb0.clone()
    api.gemm(qa, qb, alpha=-2.0, accumulate=True, out=cb)
    torch.cuda.synchronize()
    ratio = gemm_check(cb.float().cpu().numpy(), ah, bh, alpha=-2.0, c0=cb0.float().cpu().numpy(), bf16=True)
    assert ratio <= 1.0, ratio


def test_gemm_strided_output_and_zero_operand():
    M, N, K = 256, 256, 256
    a, b = operands(M, N, K, seed=3)
    qa, qb, ah, bh = quantised_pair(a, b)
    big = torch.full((M, N + 64), 7.0, device="cuda")
    out = big[:, :N]
    api.gemm(qa, qb, out_dtype=torch.float32, out=out)
    torch.cuda.synchronize()
    assert gemm_check(out.cpu().numpy(), ah, bh) <= 1.0
    assert torch.all(big[:, N:] == 7.0)
    z = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    qz, _ = api.quantize(z)
    cz = api.gemm(qz, qb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.count_nonzero(cz) == 0


def test_gemm_large_k_accumulation():
    # K = 16384: the FP32 tensor-memory accumulation over 256 MMA k-steps
    M, N, K = 256, 256, 16384
    a, b = operands(M, N, K, seed=21)
    qa, qb, ah, bh = quantised_pair(a, b)
    c = api.gemm(qa, qb, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ratio = gemm_check(c.cpu().numpy(), ah, bh)
    assert ratio <= 1.0, ratio


def test_status_clean_after_gemms():
    api.get_status()


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_accumulate_multiwave(out_dtype):
    """C += alpha * A . B^T over many persistent tiles (2304 x 3200: 9 x 12.5 tiles of
    256 x 256, a ragged raster group and a 128-column N tail), every element checked."""
    M, N, K = 2304, 3200, 512
    a, b = operands(M, N, K, seed=77)
    qa, qb, ah, bh = quantised_pair(a, b)
    g = torch.Generator(device="cuda").manual_seed(9)
    c0 = (torch.randn((M, N), generator=g, device="cuda") * 4).to(out_dtype)
    c = c0.clone()
    api.gemm(qa, qb, alpha=-0.5, accumulate=True, out=c)
    torch.cuda.synchronize()
    ratio = gemm_check(c.float().cpu().numpy(), ah, bh, alpha=-0.5, c0=c0.float().cpu().numpy(),
                       bf16=out_dtype == torch.bfloat16)
    assert ratio <= 1.0, ratio
    api.get_status()


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_grouped_mixed_shapes(out_dtype):
    """One grouped launch over problems of different M, N and K (K tails, an N tail, a
    half-empty row block, a single-row-block problem): every output within the bound of
    the oracle, and equal bit for bit to a single launch of the same pair kernel where
    that launch exists (M >= 256; a 128-row single GEMM takes the single-CTA kernel)."""
    shapes = [(512, 384, 576), (384, 256, 1088), (256, 640, 64), (128, 256, 320), (768, 128, 832)]
    problems, refs = [], []
    for i, (M, N, K) in enumerate(shapes):
        a, b = operands(M, N, K, seed=100 + i, kind="t" if i % 2 else "outliers")
        qa, qb, ah, bh = quantised_pair(a, b)
        problems.append((qa, qb))
        refs.append((ah, bh))
    outs = api.gemm_grouped(problems, out_dtype=out_dtype)
    api.get_status()
    bf16 = out_dtype == torch.bfloat16
    for (M, N, K), (qa, qb), (ah, bh), c in zip(shapes, problems, refs, outs):
        ratio = gemm_check(c.float().cpu().numpy(), ah, bh, bf16=bf16)
        assert ratio <= 1.0, ((M, N, K), ratio)
        if M >= 256:
            single = api.gemm(qa, qb, out_dtype=out_dtype)
            assert torch.equal(c, single), (M, N, K)


def test_gemm_matches_library_nvfp4_bit_for_bit():
    """Cross-check with an independent implementation: the library NVFP4 GEMM
    (torch._scaled_mm on FP4 operands with E4M3 block scales, cuBLASLt) fed the same
    quantised operands -- our codes, and our block scales, whose tensor-core layout is
    the library's swizzled layout -- gives an FP32 product that, times S_A * S_B, equals
    this library's FP32 output bit for bit at the 12B up-projection shape."""
    M, N, K = 16384, 20480, 5120
    a = synthetic.normal((M, K), 1.0, seed=30, device="cuda")
    b = synthetic.normal((N, K), 1.0, seed=31, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    del a, b
    try:
        ref = torch._scaled_mm(qa.codes.view(torch.float4_e2m1fn_x2), qb.codes.view(torch.float4_e2m1fn_x2).t(),
                               qa.scales.view(torch.float8_e4m3fn).reshape(-1),
                               qb.scales.view(torch.float8_e4m3fn).reshape(-1), out_dtype=torch.float32)
    except (RuntimeError, TypeError, AttributeError) as e:
        pytest.skip("library NVFP4 GEMM unavailable: %s" % str(e)[:120])
    ours = api.gemm(qa, qb, out_dtype=torch.float32)
    api.get_status()
    g = qa.tensor_scale * qb.tensor_scale          # FP32 product of the two tensor scales
    assert torch.equal(ours, ref * g)
