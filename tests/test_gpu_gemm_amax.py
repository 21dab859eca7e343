"""GPU parity of nvfp4_gemm_amax: the GEMM epilogue reporting the maxima that the next
quantisation of its output needs (max |C| and max |RHT16 col(C)|).

Exact construction: operand values code * u (u per 16-block in {1/8, 1/4, 1/2}, one
block per tensor at u = 7/8 holding +-5.25, every block holding a +-6 code) make both
tensor scales 2^-9 and every block scale a power of two or 448, so the oracle's
dequantised operands equal the inputs, every partial sum of the FP32 accumulation is
exact, and the BF16 output is the round-to-nearest-even of the oracle's exact FP64
product.  The oracle therefore predicts C bit for bit, and from it both maxima and
the quantisation of C that uses them.
"""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import assert_layout_equal, bf16_to_np, exact_operand

pytestmark = pytest.mark.gpu

SIGNS = 0x5A3C


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (512, 384, 512), (768, 640, 1024)])
def test_gemm_amax_exact(M, N, K):
    a, ah = exact_operand(M, K, M + K)
    b, bh = exact_operand(N, K, N + K + 1)
    ra, rb = O.quantize(ah)["row"], O.quantize(bh)["row"]
    assert ra[2] == np.float32(2.0 ** -9) and rb[2] == np.float32(2.0 ** -9)
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    assert_layout_equal(qa, ra, "A")
    assert_layout_equal(qb, rb, "B")

    c_ref = O.gemm_ref(O.dequantize(*ra), O.dequantize(*rb))                # exact in FP64
    c_bits = O.f32_to_bf16_bits(c_ref.astype(np.float32))
    c_exp = O.bf16_bits_to_f32(c_bits)

    c, amax = api.gemm_amax(qa, qb, rht_signs=SIGNS)
    got_bits = c.view(torch.int16).cpu().numpy().astype(np.uint16)
    assert (got_bits == c_bits).all(), "C differs from the exact product rounded to BF16"

    want_raw = np.float32(np.abs(c_exp).max())
    want_rht = O.transformed_amax(np.ascontiguousarray(c_exp.T), True, SIGNS)
    got = amax.cpu().numpy()
    assert got[0].view(np.uint32) == want_raw.view(np.uint32), (got[0], want_raw)
    assert got[1].view(np.uint32) == np.float32(want_rht).view(np.uint32), (got[1], want_rht)
    assert got[2] == 0.0

    # the next quantisation of C with these maxima: bit-identical to the oracle's own
    rq, cq = api.quantize(c, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS, amax_in=amax)
    ref = O.quantize(c_exp, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS)
    assert_layout_equal(rq, ref["row"], "C row")
    assert_layout_equal(cq, ref["col"], "C col (RHT)")


def test_gemm_amax_matches_amax_pass_at_full_size():
    """The 12B hybrid up-projection fprop (16384 x 20480 x 5120): the epilogue's maxima equal
    those of the quantiser's own amax pass over the same C (itself checked against the
    oracle elsewhere), and C equals nvfp4_gemm's output."""
    x = synthetic.normal((16384, 5120), 1.0, seed=12, device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    w = synthetic.normal((20480, 5120), 0.014, seed=10, device="cuda")
    qx, _ = api.quantize(x)
    qw, _ = api.quantize_weight(w)
    y_plain = api.gemm(qx, qw)
    y, amax = api.gemm_amax(qx, qw, rht_signs=SIGNS)
    assert torch.equal(y.view(torch.int16), y_plain.view(torch.int16))
    pass_amax = torch.zeros(3, dtype=torch.float32, device="cuda")
    api.quantize(y, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS, amax_out=pass_amax)
    got, want = amax.cpu().numpy(), pass_amax.cpu().numpy()
    assert got[0].view(np.uint32) == want[0].view(np.uint32), (got, want)
    assert got[1].view(np.uint32) == want[1].view(np.uint32), (got, want)


def test_gemm_amax_rejects_small_m():
    a = synthetic.normal((128, 256), 1.0, seed=1, device="cuda")
    b = synthetic.normal((256, 256), 1.0, seed=2, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    with pytest.raises(api.NVFP4Error):
        api.gemm_amax(qa, qb)
