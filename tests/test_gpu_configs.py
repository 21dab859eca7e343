"""GPU parity on the named workloads that the other files do not cover whole.

  * tiny quantise + GEMM: A, B [256 x 256] ~ N(0,1) with 1 % outliers x50 (seeds 0
    and 100), 1x16 round-to-nearest quantisation of both, C = A . B^T: codes, scales
    and tensor scales bit-exact, the whole C within the GEMM bound (FP32 output) and
    within the bound plus one BF16 half-ulp (BF16 output);
  * quantiser sweep at 4096 x 4096 (Student-t, nu = 3, x 0.1): every byte of both
    layouts in the three modes (1D RNE, 1D SR + RHT, 2D 16 x 16 blocks);
  * whole-output GEMMs over many persistent tiles: 4096 x 4096 x 1024 (256 output
    tiles of 256 x 256 on at most 74 CTA pairs, so every pair runs several tiles
    and flips its accumulator phase) and 2304 x 3200 x 512 (9 row blocks, so the
    raster group of 16 row blocks is ragged, and a 128-column N tail);
  * the square GEMM sweep: 4096^3 whole, 8192^3, 16384^3 and 32768^3 on sampled
    rows and columns (codes and scales of the sampled rows bit-exact).
"""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import assert_layout_equal, bf16_to_np, gemm_check
from tests.test_gpu_fullsize import check_gemm, check_rows, host_f32, raw_amax, sample_rows

pytestmark = pytest.mark.gpu

SIGNS, SEED = 0x5A3C, 1234


def test_tiny_config_whole():
    a, b = synthetic.tiny(device="cuda")
    ah_in, bh_in = bf16_to_np(a), bf16_to_np(b)
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    ra, rb = O.quantize(ah_in)["row"], O.quantize(bh_in)["row"]
    assert_layout_equal(qa, ra, "A")
    assert_layout_equal(qb, rb, "B")
    ah, bh = O.dequantize(*ra), O.dequantize(*rb)
    c32 = api.gemm(qa, qb, out_dtype=torch.float32)
    c16 = api.gemm(qa, qb, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert gemm_check(c32.cpu().numpy(), ah, bh) <= 1.0
    assert gemm_check(c16.float().cpu().numpy(), ah, bh, bf16=True) <= 1.0
    api.get_status()


SWEEP_MODES = {
    "rne": dict(),
    "sr_rht": dict(stochastic=True, rht_row=True, rht_col=True, seed=SEED, rht_signs=SIGNS),
    "2d": dict(block_2d=True),
}


@pytest.mark.parametrize("mode", list(SWEEP_MODES))
def test_quantizer_sweep_4096_whole(mode):
    x = synthetic.qsweep(4096, device="cuda")
    kw = SWEEP_MODES[mode]
    rq, cq = api.quantize(x, emit_row=True, emit_col=True, **kw)
    ref = O.quantize(bf16_to_np(x), emit_row=True, emit_col=True, **kw)
    assert_layout_equal(rq, ref["row"], mode + " row")
    assert_layout_equal(cq, ref["col"], mode + " col")
    api.get_status()


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 1024), (2304, 3200, 512)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_multiwave_gemm_whole_output(M, N, K, out_dtype):
    a = synthetic.normal((M, K), 1.0, seed=M + 1, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
    b = synthetic.normal((N, K), 1.0, seed=N + 2, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    ra, rb = O.quantize(bf16_to_np(a))["row"], O.quantize(bf16_to_np(b))["row"]
    assert_layout_equal(qa, ra, "A")
    assert_layout_equal(qb, rb, "B")
    c = api.gemm(qa, qb, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ratio = gemm_check(c.float().cpu().numpy(), O.dequantize(*ra), O.dequantize(*rb),
                       bf16=out_dtype == torch.bfloat16)
    assert ratio <= 1.0, ratio
    api.get_status()


def test_square_gemm_4096_whole():
    a, b = synthetic.square(4096, 0, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    ra, rb = O.quantize(bf16_to_np(a))["row"], O.quantize(bf16_to_np(b))["row"]
    assert_layout_equal(qa, ra, "A")
    assert_layout_equal(qb, rb, "B")
    c = api.gemm(qa, qb)
    torch.cuda.synchronize()
    assert gemm_check(c.float().cpu().numpy(), O.dequantize(*ra), O.dequantize(*rb), bf16=True) <= 1.0
    api.get_status()


def chunked_amax(x, rows=2048):
    """max |x| over a large BF16 device tensor, taken on the host a block of rows at a time."""
    return np.float32(max(raw_amax(host_f32(x[r0:r0 + rows])) for r0 in range(0, x.shape[0], rows)))


@pytest.mark.parametrize("i,n", [(1, 8192), (2, 16384), (3, 32768)])
def test_square_gemm_sampled(i, n):
    """M = N = K = n, BF16 output, as bench.py --kernel gemm launches it."""
    a, b = synthetic.square(n, i, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    c = api.gemm(qa, qb)
    api.get_status()
    ra_rows, rb_rows = sample_rows(n, 500 + i), sample_rows(n, 600 + i)
    a_rows = host_f32(a[torch.as_tensor(ra_rows, device="cuda")])
    b_rows = host_f32(b[torch.as_tensor(rb_rows, device="cuda")])
    S_a = O.tensor_scale(chunked_amax(a))
    S_b = O.tensor_scale(chunked_amax(b))
    del a, b
    codes, scales = O.quantize_layout_rows(a_rows, ra_rows, n, S_a, rht=False, signs=0, stochastic=False,
                                           seed=0, offset=0, tag=0)
    a_hat = check_rows(qa, ra_rows, codes, scales, S_a, "A rows")
    codes, scales = O.quantize_layout_rows(b_rows, rb_rows, n, S_b, rht=False, signs=0, stochastic=False,
                                           seed=0, offset=0, tag=0)
    b_hat = check_rows(qb, rb_rows, codes, scales, S_b, "B rows")
    check_gemm(c, ra_rows, rb_rows, a_hat, b_hat, "square %d^3" % n)
    del c, qa, qb
    torch.cuda.empty_cache()


def test_layer3b_grouped_wgrad_matches_separate_launches():
    """The four weight-gradient GEMMs of the 3B decoder layer at 32768 tokens (QKV, O,
    gate-up, down) in one grouped launch give, tile for tile, the same FP32 outputs as
    four separate launches (bit for bit: the same accumulation order in every tile), and
    sampled rows of each agree with the oracle within the GEMM bound."""
    import bench
    from tests.test_gpu_fullsize import host_f32, layout_rows_1d, check_rows
    names = list(synthetic.LAYER3B["linears"])
    problems, singles, refs = [], [], []
    for i, name in enumerate(names):
        x, w, dy = synthetic.layer3b_linear(name, device="cuda")
        _, xc = api.quantize(x, emit_row=False, emit_col=True, rht_col=True, rht_signs=bench.RHT_SIGNS)
        _, dc = api.quantize(dy, emit_row=False, emit_col=True, stochastic=True, rht_col=True, seed=bench.SR_SEED,
                             rht_signs=bench.RHT_SIGNS)
        problems.append((dc, xc))
        singles.append(api.gemm(dc, xc, out_dtype=torch.float32))
        if name == "o":
            refs.append((name, x, dy, dc, xc))
        del x, w, dy
    outs = api.gemm_grouped(problems, out_dtype=torch.float32)
    api.get_status()
    for name, a, b in zip(names, outs, singles):
        assert torch.equal(a, b), name
    # the O projection's dW rows against the oracle: dY^T X over 32768 tokens
    name, x, dy, dc, xc = refs[0]
    xh, dyh = host_f32(x), host_f32(dy)
    n_rows, k_rows = sample_rows(dyh.shape[1], 700)[:8], sample_rows(xh.shape[1], 701)[:8]
    S_dc = np.float32(dc.tensor_scale.cpu().item())
    S_xc = np.float32(xc.tensor_scale.cpu().item())
    c, s = layout_rows_1d(dyh, n_rows, S_dc, col=True, rht=True, stochastic=True, seed=bench.SR_SEED, offset=0,
                          signs=bench.RHT_SIGNS)
    a_hat = check_rows(dc, n_rows, c, s, S_dc, "dY col")
    c, s = layout_rows_1d(xh, k_rows, S_xc, col=True, rht=True, stochastic=False, signs=bench.RHT_SIGNS)
    b_hat = check_rows(xc, k_rows, c, s, S_xc, "X col")
    got = outs[names.index("o")][torch.as_tensor(n_rows, device="cuda")][:, torch.as_tensor(k_rows, device="cuda")]
    ref = O.gemm_ref(a_hat, b_hat)
    ratio = np.abs(got.cpu().numpy().astype(np.float64) - ref) / O.gemm_tolerance(a_hat, b_hat)
    assert ratio.max() <= 1.0, float(ratio.max())
