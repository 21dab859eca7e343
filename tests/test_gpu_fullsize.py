"""GPU parity at the workloads' full sizes, in the launch configuration bench.py times.

The oracle cannot quantise or multiply these tensors whole in a test's time, so each
check takes what the oracle can compute one piece at a time:
  * tensor scales: the oracle's amax over the whole tensor (raw, and over the
    RHT-transformed column layout, computed in column chunks) -> S, bit-exact;
  * codes and block scales: sampled rows of every emitted layout (first, last and
    seeded random rows), quantised by the oracle from the same input rows, with
    the Philox element indices of the full layout, bit-exact;
  * GEMM outputs: every pair of sampled rows, C_ref[i, j] in FP64 from the oracle's
    dequantised rows, within the GEMM bound (BF16 output: plus one BF16 half-ulp).
Workloads: the 12B hybrid MLP step that bench.py times (both linears, all six
GEMMs), the 3B MLP step, the four linears of the 3B decoder layer (32768 tokens), and
the 8192^2 and 16384^2 quantiser sweep tensors in their three modes.
"""

import numpy as np
import pytest
import torch

import bench
from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import mma_scale_offsets

pytestmark = pytest.mark.gpu

N_RANDOM_ROWS = 12


def sample_rows(n, seed):
    rng = np.random.default_rng(seed)
    rows = set([0, 1, n - 2, n - 1]) | set(int(r) for r in rng.integers(0, n, N_RANDOM_ROWS))
    return np.array(sorted(rows), dtype=np.int64)


def host_f32(x):
    return x.float().cpu().numpy()


def raw_amax(xh):
    return np.float32(np.abs(xh).max())


def rht_col_amax(xh, signs, chunk=512):
    """amax over the RHT-transformed column layout (blocks of 16 along the first axis)."""
    best = np.float32(0.0)
    for c0 in range(0, xh.shape[1], chunk):
        best = max(best, O.transformed_amax(np.ascontiguousarray(xh[:, c0:c0 + chunk].T), True, signs))
    return np.float32(best)


def gpu_rows(q, rows):
    """(codes [n, cols/2], row-major scales [n, cols/16], S) of selected rows of a QTensor."""
    torch.cuda.synchronize()
    half = q.cols // 2
    codes = q.codes.view(q.rows, half)[torch.as_tensor(rows, device=q.codes.device)].cpu().numpy()
    buf = q.scales.cpu().numpy()
    nb = q.cols // 16
    if q.scale_layout == 1:
        offs = np.concatenate([mma_scale_offsets(128, q.cols)[r % 128][None, :] + (r // 128) * ((nb + 3) // 4) * 512
                               for r in rows])
    else:
        offs = rows[:, None] * nb + np.arange(nb)[None, :]
    return codes, buf[offs], np.float32(q.tensor_scale.cpu().item())


def check_rows(q, rows, ref_codes, ref_scales, ref_S, what):
    codes, scales, S = gpu_rows(q, rows)
    assert S.view(np.uint32) == np.float32(ref_S).view(np.uint32), (what, "tensor scale", S, ref_S)
    packed = O.pack_codes(ref_codes)
    bad = np.argwhere(scales != ref_scales)
    assert bad.size == 0, (what, "scales differ", rows[bad[0][0]], bad[:3])
    bad = np.argwhere(codes != packed)
    assert bad.size == 0, (what, "codes differ", rows[bad[0][0]], bad[:3])
    return O.dequantize(packed, ref_scales, ref_S)


def layout_rows_1d(xh, rows, S, *, col, rht, stochastic, seed=0, offset=0, signs=0):
    """Oracle rows of a 1x16 layout of xh: rows of xh (row layout) or columns (col layout)."""
    v = np.ascontiguousarray(xh[:, rows].T) if col else xh[rows]
    n_cols = xh.shape[0] if col else xh.shape[1]
    return O.quantize_layout_rows(v, rows, n_cols, S, rht=rht, signs=signs, stochastic=stochastic,
                                  seed=seed, offset=offset, tag=1 if col else 0)


def layout_rows_2d(wh, rows, amax, *, col):
    """Oracle rows of the 16x16-block layouts of a weight: each sampled row from its 16-row
    (row layout) or 16-column (col layout) strip, quantised with the whole tensor's amax."""
    codes, scales = [], []
    S = O.tensor_scale(amax)
    for r in rows:
        s0 = (r // 16) * 16
        strip = wh[:, s0:s0 + 16] if col else wh[s0:s0 + 16]
        out = O.quantize(np.ascontiguousarray(strip), emit_row=not col, emit_col=col, block_2d=True,
                         amax_in=(amax, amax))["col" if col else "row"]
        codes.append(O.unpack_codes(out[0])[r - s0])
        scales.append(out[1][r - s0])
    return np.stack(codes), np.stack(scales), S


def check_gemm(c, rows_a, rows_b, a_hat, b_hat, what):
    """Sampled C[rows_a, rows_b] (BF16) against the oracle's FP64 product of the rows."""
    torch.cuda.synchronize()
    ra = torch.as_tensor(rows_a, device=c.device)
    rb = torch.as_tensor(rows_b, device=c.device)
    got = c[ra][:, rb].float().cpu().numpy().astype(np.float64)
    ref = O.gemm_ref(a_hat, b_hat)
    bound = O.gemm_tolerance(a_hat, b_hat) + 2.0 ** -8 * np.abs(ref)
    ratio = float((np.abs(got - ref) / bound).max())
    assert ratio <= 1.0, (what, "worst |err| / bound", ratio)


def check_linear_step(L, offset, seed):
    """One bench step on linear L, then parity of all its quantised layouts and GEMMs."""
    bench.instrumented_step([L], bench.PhaseEvents(False), offset)
    api.get_status()
    M, K, N = L.M, L.K, L.N
    xh, wh, dyh = host_f32(L.x), host_f32(L.w), host_f32(L.dy)
    signs = bench.RHT_SIGNS
    ti, nj, kk = sample_rows(M, seed), sample_rows(N, seed + 1), sample_rows(K, seed + 2)

    a_x, a_w, a_dy = raw_amax(xh), raw_amax(wh), raw_amax(dyh)
    S_x, S_dy = O.tensor_scale(a_x), O.tensor_scale(a_dy)
    S_xc, S_dyc = O.tensor_scale(rht_col_amax(xh, signs)), O.tensor_scale(rht_col_amax(dyh, signs))

    c, s = layout_rows_1d(xh, ti, S_x, col=False, rht=False, stochastic=False)
    x_row = check_rows(L.xq_row, ti, c, s, S_x, "X row")
    c, s = layout_rows_1d(xh, kk, S_xc, col=True, rht=True, stochastic=False, signs=signs)
    x_col = check_rows(L.xq_col, kk, c, s, S_xc, "X col (RHT)")
    c, s, S_w = layout_rows_2d(wh, nj, a_w, col=False)
    w_row = check_rows(L.wq_row, nj, c, s, S_w, "W row (2D)")
    c, s, _ = layout_rows_2d(wh, kk, a_w, col=True)
    w_col = check_rows(L.wq_col, kk, c, s, S_w, "W col (2D)")
    c, s = layout_rows_1d(dyh, ti, S_dy, col=False, rht=False, stochastic=True, seed=bench.SR_SEED, offset=offset)
    dy_row = check_rows(L.dyq_row, ti, c, s, S_dy, "dY row (SR)")
    c, s = layout_rows_1d(dyh, nj, S_dyc, col=True, rht=True, stochastic=True, seed=bench.SR_SEED,
                          offset=offset, signs=signs)
    dy_col = check_rows(L.dyq_col, nj, c, s, S_dyc, "dY col (RHT, SR)")

    check_gemm(L.y, ti, nj, x_row, w_row, "fprop Y = X W^T")
    check_gemm(L.dx, ti, kk, dy_row, w_col, "dgrad dX = dY W")
    check_gemm(L.dw, nj, kk, dy_col, x_col, "wgrad dW = dY^T X")


def test_hybrid12b_step_fullsize():
    """The 12B hybrid MLP step of bench.py (tokens 16384, hidden 5120, FFN 20480)."""
    for i, L in enumerate(bench.build_workload(torch.device("cuda"), 0)):
        check_linear_step(L, offset=0, seed=100 + 10 * i)     # rank 0's SR offset, as in bench.py
        del L
        torch.cuda.empty_cache()


def test_mlp3b_step_fullsize():
    """3B-class MLP linear step (tokens 8192, in 3072, out 8192)."""
    x, w, dy = synthetic.mlp3b(device="cuda")
    check_linear_step(bench.Linear("mlp3b", x, w, dy), offset=0, seed=200)


@pytest.mark.parametrize("name", list(synthetic.LAYER3B["linears"]))
def test_layer3b_linear_fullsize(name):
    """The four linears of the 3B decoder layer at 32768 tokens: QKV 3072 -> 9216, O
    3072 -> 3072, gate-up 3072 -> 16384, down 8192 -> 3072."""
    x, w, dy = synthetic.layer3b_linear(name, device="cuda")
    check_linear_step(bench.Linear(name, x, w, dy), offset=0, seed=300 + len(name))
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n", [8192, 16384])
@pytest.mark.parametrize("mode", ["rne", "sr_rht", "2d"])
def test_quantizer_sweep_sampled(n, mode):
    """Quantiser sweep tensor n x n (Student-t, nu = 3, x 0.1), with the col layout."""
    x = synthetic.qsweep(n, device="cuda")
    xh = host_f32(x)
    rows = sample_rows(n, 400)
    seed, offset, signs = 1234, 0, bench.RHT_SIGNS
    if mode == "2d":
        rq, cq = api.quantize(x, emit_row=True, emit_col=True, block_2d=True)
        a = raw_amax(xh)
        c, s, S = layout_rows_2d(xh, rows, a, col=False)
        check_rows(rq, rows, c, s, S, "2D row")
        c, s, S = layout_rows_2d(xh, rows, a, col=True)
        check_rows(cq, rows, c, s, S, "2D col")
        return
    sr = mode == "sr_rht"
    rq, cq = api.quantize(x, emit_row=True, emit_col=True, stochastic=sr, rht_row=sr, rht_col=sr, seed=seed,
                          offset=offset, rht_signs=signs)
    if sr:
        S_r = O.tensor_scale(np.float32(max(O.transformed_amax(xh[r0:r0 + 1024], True, signs)
                                            for r0 in range(0, n, 1024))))
        S_c = O.tensor_scale(rht_col_amax(xh, signs))
    else:
        S_r = S_c = O.tensor_scale(raw_amax(xh))
    c, s = layout_rows_1d(xh, rows, S_r, col=False, rht=sr, stochastic=sr, seed=seed, offset=offset, signs=signs)
    check_rows(rq, rows, c, s, S_r, mode + " row")
    c, s = layout_rows_1d(xh, rows, S_c, col=True, rht=sr, stochastic=sr, seed=seed, offset=offset, signs=signs)
    check_rows(cq, rows, c, s, S_c, mode + " col")
