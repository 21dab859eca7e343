"""Test helpers: move data between torch and the oracle, and read the stored
layouts documented in include/nvfp4.h (pure index arithmetic, no quantisation)."""

import numpy as np
import torch

from oracle import nvfp4_oracle as O


def bf16_to_np(x: torch.Tensor) -> np.ndarray:
    """BF16 tensor -> float32 numpy array (exact)."""
    return x.detach().float().cpu().numpy()


def mma_scale_offsets(rows, cols):
    """Byte offset of block scale (r, j) in the tensor-core scale layout of include/nvfp4.h."""
    nb = cols // 16
    kg = (nb + 3) // 4
    r = np.arange(rows, dtype=np.int64)[:, None]
    j = np.arange(nb, dtype=np.int64)[None, :]
    return ((r // 128) * kg + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (j % 4)


def scales_rowmajor(q) -> np.ndarray:
    """Scales of a QTensor as a [rows, cols/16] uint8 array."""
    buf = q.scales.cpu().numpy()
    if q.scale_layout == 1:
        return buf[mma_scale_offsets(q.rows, q.cols)]
    return buf[: q.rows * (q.cols // 16)].reshape(q.rows, q.cols // 16)


def qtensor_np(q):
    """(packed codes, row-major scales, tensor scale) of a QTensor."""
    torch.cuda.synchronize()
    return q.codes.cpu().numpy(), scales_rowmajor(q), np.float32(q.tensor_scale.cpu().item())


def assert_layout_equal(q, ref, what=""):
    codes, scales, S = qtensor_np(q)
    rc, rs, rS = ref
    assert np.float32(S).view(np.uint32) == np.float32(rS).view(np.uint32), (what, "tensor scale", S, rS)
    bad_s = np.argwhere(scales != rs)
    assert bad_s.size == 0, (what, "scales differ at", bad_s[:5], scales[tuple(bad_s[0])], rs[tuple(bad_s[0])])
    bad_c = np.argwhere(codes != rc)
    assert bad_c.size == 0, (what, "codes differ at", bad_c[:5], codes[tuple(bad_c[0])], rc[tuple(bad_c[0])])


def gemm_check(c_gpu: np.ndarray, a_hat, b_hat, alpha=1.0, c0=None, bf16=False):
    """|C - C_ref| <= 1e-5 sum|a b| + 1e-6 (+ one BF16 half-ulp of |C_ref| for BF16 output).

    Returns the worst ratio |err| / bound (<= 1 passes)."""
    ref = O.gemm_ref(a_hat, b_hat, alpha)
    if c0 is not None:
        ref = ref + c0.astype(np.float64)
    bound = O.gemm_tolerance(a_hat, b_hat, alpha)
    if bf16:
        bound = bound + 2.0 ** -8 * np.abs(ref)
        if c0 is not None:
            bound = bound + 2.0 ** -8 * np.abs(c0.astype(np.float64))
    err = np.abs(c_gpu.astype(np.float64) - ref)
    ratio = float((err / bound).max()) if err.size else 0.0
    return ratio
