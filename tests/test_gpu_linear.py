"""GPU parity of the NVFP4 linear layer (fprop, dgrad, wgrad) against the oracle:
the quantised operands must be bit-identical and each GEMM within the bound."""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import assert_layout_equal, bf16_to_np, gemm_check

pytestmark = pytest.mark.gpu

SIGNS = 0x5A3C
SEED = 1234


def layer(M, K, N, seeds=(2, 3, 4)):
    x = synthetic.normal((M, K), 1.0, seed=seeds[0], device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    w = synthetic.normal((N, K), 0.02, seed=seeds[1], device="cuda")
    dy = synthetic.normal((M, N), 1e-3, seed=seeds[2], device="cuda")
    return x, w, dy


@pytest.mark.parametrize("M,K,N", [(256, 256, 256), (384, 384, 640), (512, 1024, 768)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_linear_step_matches_oracle(M, K, N, out_dtype):
    x, w, dy = layer(M, K, N)
    wq_row, wq_col = api.quantize_weight(w)
    y, xq_row, xq_col = api.linear_fwd(x, wq_row, rht_signs=SIGNS, out_dtype=out_dtype)
    dx, dyq_row, dyq_col = api.linear_dgrad(dy, wq_col, seed=SEED, offset=3, rht_signs=SIGNS, out_dtype=out_dtype)
    dw = api.linear_wgrad(dyq_col, xq_col, out_dtype=out_dtype)
    torch.cuda.synchronize()

    wq = O.quantize_weight(bf16_to_np(w))
    assert_layout_equal(wq_row, wq["row"], "Wq row")
    assert_layout_equal(wq_col, wq["col"], "Wq col")
    y_ref, (ah, bh), xq = O.linear_fwd_ref(bf16_to_np(x), wq, rht_signs=SIGNS)
    assert_layout_equal(xq_row, xq["row"], "Xq row")
    assert_layout_equal(xq_col, xq["col"], "Xq col")
    bf16 = out_dtype == torch.bfloat16
    assert gemm_check(y.float().cpu().numpy(), ah, bh, bf16=bf16) <= 1.0

    dx_ref, (ah, bh), dyq = O.linear_dgrad_ref(bf16_to_np(dy), wq, seed=SEED, offset=3, rht_signs=SIGNS)
    assert_layout_equal(dyq_row, dyq["row"], "dYq row")
    assert_layout_equal(dyq_col, dyq["col"], "dYq col")
    assert gemm_check(dx.float().cpu().numpy(), ah, bh, bf16=bf16) <= 1.0

    dw_ref, (ah, bh) = O.linear_wgrad_ref(dyq, xq)
    assert gemm_check(dw.float().cpu().numpy(), ah, bh, bf16=bf16) <= 1.0


def test_wgrad_accumulates_fp32():
    M, K, N = 256, 256, 384
    x, w, dy = layer(M, K, N, seeds=(5, 6, 7))
    wq_row, wq_col = api.quantize_weight(w)
    _, _, xq_col = api.linear_fwd(x, wq_row, rht_signs=SIGNS)
    _, _, dyq_col = api.linear_dgrad(dy, wq_col, seed=SEED, rht_signs=SIGNS)
    acc = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    api.linear_wgrad(dyq_col, xq_col, out=acc, accumulate=True)
    api.linear_wgrad(dyq_col, xq_col, out=acc, accumulate=True)
    one = api.linear_wgrad(dyq_col, xq_col, out_dtype=torch.float32)
    torch.cuda.synchronize()
    torch.testing.assert_close(acc, 2 * one, rtol=1e-6, atol=1e-9)


def test_rht_cancels_in_wgrad():
    """Without quantisation error the transformed wgrad equals dY^T X; with it, the
    NVFP4 wgrad stays close to the exact product."""
    M, K, N = 512, 256, 256
    x, w, dy = layer(M, K, N, seeds=(8, 9, 10))
    wq_row, wq_col = api.quantize_weight(w)
    _, _, xq_col = api.linear_fwd(x, wq_row, rht_signs=SIGNS)
    _, _, dyq_col = api.linear_dgrad(dy, wq_col, seed=SEED, rht_signs=SIGNS)
    dw = api.linear_wgrad(dyq_col, xq_col, out_dtype=torch.float32)
    exact = dy.double().t() @ x.double()
    rel = (dw.double() - exact).norm() / exact.norm()
    assert rel < 0.2, float(rel)
