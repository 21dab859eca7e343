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


E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def exact_operand(rows, cols, seed, device="cuda"):
    """A BF16 matrix that NVFP4 holds exactly: values code * u, u per 16-block in
    {1/8, 1/4, 1/2}, one block per tensor at u = 7/8 holding +-5.25, every block holding
    a +-6 code.  The tensor scale is then 2^-9 and every block scale a power of two or
    448, so dequantisation returns the input and products of such matrices have few
    significant bits.  Returns (BF16 tensor on device, float32 numpy values)."""
    rng = np.random.default_rng(seed)
    v = E2M1_GRID[rng.integers(0, 8, (rows, cols))] * rng.choice([-1.0, 1.0], (rows, cols))
    blocks = v.reshape(rows, cols // 16, 16)
    blocks[:, :, 0] = 6.0 * rng.choice([-1.0, 1.0], (rows, cols // 16))      # every block max is 6u
    u = rng.choice([0.125, 0.25, 0.5], (rows, cols // 16))
    u[rng.integers(0, rows), rng.integers(0, cols // 16)] = 0.875              # tensor amax 5.25 -> S = 2^-9
    x = (blocks * u[:, :, None]).reshape(rows, cols)
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(device), x.astype(np.float32)
