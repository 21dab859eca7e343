"""GPU parity of the quantiser (nvfp4_quantize) and dequantiser against the CPU
oracle: codes, block scales and tensor scales must be bit-identical."""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import assert_layout_equal, bf16_to_np, qtensor_np

pytestmark = pytest.mark.gpu

SHAPES = [(256, 256), (48, 96), (400, 288), (1040, 800), (128, 4096)]
MODES = {
    "rne_row": dict(emit_row=True),
    "rne_row_col": dict(emit_row=True, emit_col=True),
    "rne_row_rhtcol": dict(emit_row=True, emit_col=True, rht_col=True),            # activations (fprop + wgrad)
    "sr_row_rhtcol": dict(emit_row=True, emit_col=True, stochastic=True, rht_col=True),  # gradients
    "sr_rht_both": dict(emit_row=True, emit_col=True, stochastic=True, rht_row=True, rht_col=True),
    "sr_row": dict(emit_row=True, stochastic=True),
    "rne_rhtrow": dict(emit_row=True, rht_row=True),
    "col_only_sr": dict(emit_row=False, emit_col=True, stochastic=True),
    "2d": dict(emit_row=True, emit_col=True, block_2d=True),
}


def _inputs(shape, kind, seed=0):
    if kind == "normal_outliers":
        return synthetic.normal(shape, 1.0, seed=seed, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
    if kind == "student_t":
        return synthetic.student_t(shape, 3, 0.1, seed=seed, device="cuda")
    if kind == "tiny":
        return synthetic.normal(shape, 1e-38, seed=seed, device="cuda")
    raise ValueError(kind)


def run_both(x, mode, layout=api.SCALE_MMA, seed=1234, offset=7, signs=0xA53C):
    kw = dict(MODES[mode])
    kw.setdefault("emit_row", True)
    rq, cq = api.quantize(x, seed=seed, offset=offset, rht_signs=signs, scale_layout=layout, **kw)
    ref = O.quantize(bf16_to_np(x), seed=seed, offset=offset, rht_signs=signs, **kw)
    return rq, cq, ref


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("mode", list(MODES))
def test_quantize_matches_oracle(shape, mode):
    x = _inputs(shape, "normal_outliers", seed=shape[0] + shape[1])
    rq, cq, ref = run_both(x, mode)
    if rq is not None:
        assert_layout_equal(rq, ref["row"], mode + " row")
    if cq is not None:
        assert_layout_equal(cq, ref["col"], mode + " col")


@pytest.mark.parametrize("mode", ["rne_row_rhtcol", "sr_rht_both", "2d"])
def test_quantize_rowmajor_scale_layout(mode):
    x = _inputs((272, 320), "student_t", seed=5)
    rq, cq, ref = run_both(x, mode, layout=api.SCALE_ROWMAJOR)
    assert_layout_equal(rq, ref["row"], mode)
    assert_layout_equal(cq, ref["col"], mode)


@pytest.mark.parametrize("kind", ["student_t", "tiny"])
def test_quantize_distributions(kind):
    x = _inputs((512, 512), kind, seed=3)
    for mode in ("sr_rht_both", "2d", "rne_row_col"):
        rq, cq, ref = run_both(x, mode)
        assert_layout_equal(rq, ref["row"], mode)
        assert_layout_equal(cq, ref["col"], mode)


def test_quantize_edge_values():
    g = torch.Generator(device="cuda").manual_seed(9)
    x = torch.randn((256, 512), generator=g, device="cuda")
    x[0, :16] = 0.0                                  # an all-zero block
    x[1, :16] = -0.0                                 # negative zeros
    x[2, 5] = 3e38                                   # huge outlier
    x[3, :] = 1e-40                                  # subnormal BF16 values
    x[4, 16:32] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 2) * 448 / 6
    x[5:21, 32:48] = 0.0                             # an all-zero 16x16 tile
    x = x.to(torch.bfloat16)
    for mode in ("rne_row_col", "sr_rht_both", "2d", "rne_row_rhtcol"):
        rq, cq, ref = run_both(x, mode)
        assert_layout_equal(rq, ref["row"], mode)
        assert_layout_equal(cq, ref["col"], mode)


def test_quantize_zero_tensor_and_empty():
    x = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    rq, cq, ref = run_both(x, "sr_rht_both")
    assert_layout_equal(rq, ref["row"])
    assert float(rq.tensor_scale.item()) == 1.0
    e = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    rq, cq = api.quantize(e, emit_row=True, emit_col=True)
    torch.cuda.synchronize()
    assert float(rq.tensor_scale.item()) == 1.0


def test_quantize_row_only_ragged_rows():
    x = _inputs((40, 272), "normal_outliers", seed=8)
    for mode in ("rne_row", "sr_row", "rne_rhtrow"):
        rq, _, ref = run_both(x, mode)
        assert_layout_equal(rq, ref["row"], mode)


def test_quantize_strided_input():
    base = _inputs((256, 640), "normal_outliers", seed=11)
    x = base[:, 64:576]                                # row stride 640 elements
    rq, cq, ref = run_both(x, "sr_rht_both")
    assert_layout_equal(rq, ref["row"])
    assert_layout_equal(cq, ref["col"])


def test_amax_in_and_out():
    x = _inputs((256, 256), "normal_outliers", seed=12)
    amax_out = torch.zeros(3, dtype=torch.float32, device="cuda")
    rq, cq = api.quantize(x, emit_row=True, emit_col=True, rht_col=True, amax_out=amax_out)
    ref = O.quantize(bf16_to_np(x), emit_row=True, emit_col=True, rht_col=True)
    torch.cuda.synchronize()
    got = amax_out.cpu().numpy()
    assert got[0] == ref["amax"][0] and got[1] == ref["amax"][1]
    # replaying with the measured maxima skips the amax pass and gives the same bytes
    rq2, cq2 = api.quantize(x, emit_row=True, emit_col=True, rht_col=True, amax_in=amax_out.clone())
    assert_layout_equal(rq2, ref["row"])
    assert_layout_equal(cq2, ref["col"])
    # a smaller external amax saturates like the oracle does
    small = torch.tensor([1.0, 1.0, 0.0], device="cuda")
    rq3, _ = api.quantize(x, emit_row=True, amax_in=small)
    ref3 = O.quantize(bf16_to_np(x), emit_row=True, amax_in=(1.0, 1.0))
    assert_layout_equal(rq3, ref3["row"])


def test_sr_reproducible_and_seed_dependent():
    x = _inputs((256, 256), "normal_outliers", seed=13)
    a, _ = api.quantize(x, stochastic=True, seed=1, offset=0)
    b, _ = api.quantize(x, stochastic=True, seed=1, offset=0)
    c, _ = api.quantize(x, stochastic=True, seed=2, offset=0)
    d, _ = api.quantize(x, stochastic=True, seed=1, offset=1)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)
    assert not torch.equal(a.codes, c.codes)
    assert not torch.equal(a.codes, d.codes)


@pytest.mark.parametrize("layout", [api.SCALE_MMA, api.SCALE_ROWMAJOR])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dequantize_matches_oracle(layout, dtype):
    x = _inputs((384, 320), "normal_outliers", seed=14)
    rq, _ = api.quantize(x, scale_layout=layout)
    out = api.dequantize(rq, dtype)
    ref = O.quantize(bf16_to_np(x))
    deq = O.dequantize(*ref["row"])
    torch.cuda.synchronize()
    if dtype == torch.float32:
        assert np.array_equal(out.cpu().numpy().view(np.uint32), deq.view(np.uint32))
    else:
        assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), O.f32_to_bf16_bits(deq))


def test_2d_weight_col_is_exact_transpose():
    w = synthetic.normal((384, 640), 0.02, seed=15, device="cuda")
    rq, cq = api.quantize_weight(w)
    rc, rs, rS = qtensor_np(rq)
    cc, cs, cS = qtensor_np(cq)
    assert rS == cS
    assert np.array_equal(O.unpack_codes(rc).T, O.unpack_codes(cc))
    assert np.array_equal(np.repeat(rs[::16, :].T, 16, axis=0), cs)


def near_midpoint_blocks(rows, cols, amax, seed):
    """BF16-valued FP32 [rows x cols] whose 16-element row blocks each have a maximum b
    close to 6 * S * m for an E4M3 rounding midpoint m (S = fl(amax / 2688), set by one
    element equal to amax): the BF16 value nearest 6 S m, or one up to 4 BF16 steps away,
    so that the block scale fl(fl(b / 6) / S) lands on or within a few FP32 ulps of the
    place where its E4M3 rounding changes."""
    rng = np.random.default_rng(seed)
    S = float(np.float32(np.float32(amax) / np.float32(2688.0)))
    mids = [(1.0 + (2 * k + 1) / 16.0) * 2.0 ** e for e in range(-6, 9) for k in range(8)]
    mids = [m for m in mids if m < 448.0] + [(k + 0.5) * 2.0 ** -9 for k in range(8)]   # + subnormal midpoints
    nb = rows * cols // 16
    x = np.empty((nb, 16), dtype=np.float32)
    for i in range(nb):
        b = O.bf16_round(np.array([6.0 * S * mids[i % len(mids)]], dtype=np.float32))
        bits = b.view(np.uint32).astype(np.int64) + 0x10000 * int(rng.integers(-4, 5))
        bb = np.array([bits[0]], dtype=np.uint32).view(np.float32)[0]
        row = np.empty(16, dtype=np.float32)
        row[0] = bb if rng.random() < 0.5 else -bb
        row[1:] = O.bf16_round((rng.uniform(-0.9, 0.9, 15) * bb).astype(np.float32))
        rng.shuffle(row)
        x[i] = row
    x = x.reshape(rows, cols)
    x[0, 0] = np.float32(amax)
    return x


@pytest.mark.parametrize("amax", [2688.0, 3008.0, 2688.0 * 2.0 ** -20, 0.01171875])
@pytest.mark.parametrize("mode", ["rne_row_col", "sr_row", "2d"])
def test_block_scales_near_e4m3_midpoints(amax, mode):
    """Block maxima whose scales sit on or next to E4M3 rounding midpoints, with tensor
    scales that are powers of two (S = 1 and 2^-20: exact ties) and general ones: the
    block scale bytes, codes and tensor scales equal the oracle's bit for bit."""
    x = torch.from_numpy(near_midpoint_blocks(256, 512, amax, seed=int(amax * 7) % 1000)).to(torch.bfloat16).cuda()
    rq, cq, ref = run_both(x, mode)
    if rq is not None:
        assert_layout_equal(rq, ref["row"], mode + " row")
    if cq is not None:
        assert_layout_equal(cq, ref["col"], mode + " col")


@pytest.mark.parametrize("above", [False, True])
@pytest.mark.parametrize("mode", ["rne_row_rhtcol", "sr_row_rhtcol", "sr_rht_both"])
def test_rht_quarter_fold_boundary(above, mode):
    """The transform's 1/4 is folded into the block maximum and the encode multiplier
    while the tensor scale S is at most 2^100, and applied to the values above it.
    Tensors with S = 2^100 exactly (maximum 2688 * 2^100) and with the next BF16
    maximum up, their values spread over 160 binades, equal the oracle bit for bit on
    both sides of the switch."""
    rng = np.random.default_rng(31 + int(above))
    x = rng.standard_normal((256, 384)) * np.exp2(rng.integers(-60, 100, (256, 384)).astype(np.float64))
    x = O.bf16_round(x.astype(np.float32))
    amax = np.array([2688.0 * 2.0 ** 100], dtype=np.float32)
    if above:
        amax = (amax.view(np.uint32) + np.uint32(0x10000)).view(np.float32)
    x[7, 9] = amax[0]
    assert np.abs(x).max() == amax[0]
    rq, cq, ref = run_both(torch.from_numpy(x).to(torch.bfloat16).cuda(), mode)
    assert_layout_equal(rq, ref["row"], mode + " row")
    assert_layout_equal(cq, ref["col"], mode + " col")
