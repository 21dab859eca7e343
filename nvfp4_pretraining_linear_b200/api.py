"""PyTorch-facing binding of the C ABI: the same entry points, with torch tensors.

Only marshalling happens here -- buffers are torch CUDA tensors, the stream is
torch's current stream, and every step of the computation runs in the CUDA
library.  There is no CPU path: calls fail when the library or a GPU is missing.
"""

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import OUT_BF16, OUT_F32, SCALE_MMA, SCALE_ROWMAJOR, NVFP4Error  # noqa: F401

_workspaces = {}

# With NVFP4_CHECK_STATUS=1 in the environment every call below synchronises its stream
# and raises on a recorded device-side error (a bounded wait that gave up), at the call
# that caused it.  Off by default: the library's calls are asynchronous, and a training
# step normally checks nvfp4_get_status once (get_status() here) before using results.
_CHECK_EACH_CALL = os.environ.get("NVFP4_CHECK_STATUS", "") not in ("", "0")


def _checked(status, stream=None):
    _lib.check(status)
    if _CHECK_EACH_CALL:
        _lib.check(_lib.load().nvfp4_get_status(_stream_ptr(stream)))


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def workspace(device=None, stream=None):
    """A cached workspace buffer per (device, stream) for the quantiser's amax pass."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev.index, s.cuda_stream)
    ws = _workspaces.get(key)
    if ws is None:
        n = _lib.load().nvfp4_workspace_size()
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
        _workspaces[key] = ws
    return ws


@dataclass
class QTensor:
    """An NVFP4 tensor: packed codes [rows, cols/2], block scales, FP32 tensor scale."""
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor
    rows: int
    cols: int
    scale_layout: int = SCALE_MMA

    def struct(self):
        return _lib.NVFP4Tensor(self.codes.data_ptr(), self.scales.data_ptr(), self.tensor_scale.data_ptr(),
                                self.rows, self.cols, self.scale_layout, 0)

    @staticmethod
    def empty(rows, cols, scale_layout=SCALE_MMA, device="cuda"):
        lib = _lib.load()
        nsc = lib.nvfp4_scales_bytes(rows, cols, scale_layout)
        return QTensor(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                       torch.zeros(max(nsc, 1), dtype=torch.uint8, device=device),
                       torch.empty(1, dtype=torch.float32, device=device), rows, cols, scale_layout)


def quantize(x: torch.Tensor, *, emit_row=True, emit_col=False, stochastic=False, rht_row=False, rht_col=False,
             block_2d=False, seed=0, offset=0, rht_signs=0, scale_layout=SCALE_MMA, amax_in=None, amax_out=None,
             out_row: Optional[QTensor] = None, out_col: Optional[QTensor] = None, stream=None):
    """nvfp4_quantize on a BF16 CUDA tensor [rows, cols] (last dim contiguous)."""
    lib = _lib.load()
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D BF16 CUDA tensor with a contiguous last dimension")
    rows, cols = x.shape
    if emit_row and out_row is None:
        out_row = QTensor.empty(rows, cols, scale_layout, x.device)
    if emit_col and out_col is None:
        out_col = QTensor.empty(cols, rows, scale_layout, x.device)
    opts = _lib.QuantOpts(int(stochastic), int(rht_row), int(rht_col), int(block_2d), seed, offset, rht_signs, 0,
                          _ptr(amax_in), _ptr(amax_out))
    ws = workspace(x.device, stream)
    rs = out_row.struct() if emit_row else None
    cs = out_col.struct() if emit_col else None
    _checked(lib.nvfp4_quantize(x.data_ptr(), rows, cols, x.stride(0), opts, rs, cs, ws.data_ptr(), ws.numel(),
                                  _stream_ptr(stream)), stream)
    return (out_row if emit_row else None), (out_col if emit_col else None)


def dequantize(q: QTensor, out_dtype=torch.float32, out: Optional[torch.Tensor] = None, stream=None):
    lib = _lib.load()
    if out is None:
        out = torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.codes.device)
    code = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _checked(lib.nvfp4_dequantize(q.struct(), out.data_ptr(), out.stride(0), code, _stream_ptr(stream)), stream)
    return out


def gemm(A: QTensor, B: QTensor, out_dtype=torch.bfloat16, alpha=1.0, accumulate=False,
         out: Optional[torch.Tensor] = None, stream=None):
    """nvfp4_gemm: C[M, N] = alpha * S_A * S_B * A . B^T (+ C)."""
    lib = _lib.load()
    if out is None:
        out = (torch.zeros if accumulate else torch.empty)((A.rows, B.rows), dtype=out_dtype, device=A.codes.device)
    code = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _checked(lib.nvfp4_gemm(A.struct(), B.struct(), out.data_ptr(), out.stride(0), code, alpha, int(accumulate),
                              _stream_ptr(stream)), stream)
    return out


def gemm_grouped(problems, out_dtype=torch.float32, outs=None, stream=None):
    """nvfp4_gemm_grouped: C_i = S_Ai S_Bi A_i . B_i^T for up to 8 (A_i, B_i) pairs in one
    persistent launch (the tiles of all problems form one queue).  Returns the outputs."""
    lib = _lib.load()
    n = len(problems)
    if outs is None:
        outs = [torch.empty((a.rows, b.rows), dtype=out_dtype, device=a.codes.device) for a, b in problems]
    code = OUT_F32 if outs[0].dtype == torch.float32 else OUT_BF16
    if any(o.dtype != outs[0].dtype for o in outs):
        raise ValueError("all outputs of a grouped GEMM have one type")
    sa = [a.struct() for a, _ in problems]
    sb = [b.struct() for _, b in problems]
    arr_a = (ctypes.POINTER(_lib.NVFP4Tensor) * n)(*[ctypes.pointer(x) for x in sa])
    arr_b = (ctypes.POINTER(_lib.NVFP4Tensor) * n)(*[ctypes.pointer(x) for x in sb])
    arr_c = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    arr_ld = (ctypes.c_int64 * n)(*[o.stride(0) for o in outs])
    _checked(lib.nvfp4_gemm_grouped(arr_a, arr_b, arr_c, arr_ld, n, code, _stream_ptr(stream)), stream)
    return outs


def gemm_amax(A: QTensor, B: QTensor, alpha=1.0, rht_signs=0, out: Optional[torch.Tensor] = None,
              amax: Optional[torch.Tensor] = None, stream=None):
    """nvfp4_gemm_amax: BF16 C = alpha * S_A * S_B * A . B^T and the maxima its next
    quantisation needs, as a 3-float device tensor usable as quantize(amax_in=...)."""
    lib = _lib.load()
    if out is None:
        out = torch.empty((A.rows, B.rows), dtype=torch.bfloat16, device=A.codes.device)
    if amax is None:
        amax = torch.empty(3, dtype=torch.float32, device=A.codes.device)
    _checked(lib.nvfp4_gemm_amax(A.struct(), B.struct(), out.data_ptr(), out.stride(0), alpha, rht_signs & 0xFFFF,
                                   amax.data_ptr(), _stream_ptr(stream)), stream)
    return out, amax


def quantize_weight(w: torch.Tensor, stream=None):
    """2D 16x16-block quantisation of a weight [N, K]: (row layout [N x K], col layout [K x N])."""
    return quantize(w, emit_row=True, emit_col=True, block_2d=True, stream=stream)


def linear_fwd(x: torch.Tensor, wq_row: QTensor, *, save_col=True, rht_signs=0, out_dtype=torch.bfloat16,
               out=None, xq_row=None, xq_col=None, stream=None):
    """nvfp4_linear_fwd: returns (Y, Xq_row, Xq_col or None)."""
    lib = _lib.load()
    M, K = x.shape
    N = wq_row.rows
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    if xq_row is None:
        xq_row = QTensor.empty(M, K, SCALE_MMA, x.device)
    if save_col and xq_col is None:
        xq_col = QTensor.empty(K, M, SCALE_MMA, x.device)
    ws = workspace(x.device, stream)
    code = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    xr = xq_row.struct()
    xc = xq_col.struct() if save_col else None
    _checked(lib.nvfp4_linear_fwd(x.data_ptr(), M, K, x.stride(0), wq_row.struct(), out.data_ptr(), out.stride(0),
                                    code, xr, xc, rht_signs, ws.data_ptr(), ws.numel(), _stream_ptr(stream)), stream)
    return out, xq_row, (xq_col if save_col else None)


def linear_dgrad(dy: torch.Tensor, wq_col: QTensor, *, seed, offset=0, save_col=True, rht_signs=0,
                 out_dtype=torch.bfloat16, out=None, dyq_row=None, dyq_col=None, stream=None):
    """nvfp4_linear_dgrad: returns (dX, dYq_row, dYq_col or None)."""
    lib = _lib.load()
    M, N = dy.shape
    K = wq_col.rows
    if out is None:
        out = torch.empty((M, K), dtype=out_dtype, device=dy.device)
    if dyq_row is None:
        dyq_row = QTensor.empty(M, N, SCALE_MMA, dy.device)
    if save_col and dyq_col is None:
        dyq_col = QTensor.empty(N, M, SCALE_MMA, dy.device)
    ws = workspace(dy.device, stream)
    code = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    dr = dyq_row.struct()
    dc = dyq_col.struct() if save_col else None
    _checked(lib.nvfp4_linear_dgrad(dy.data_ptr(), M, N, dy.stride(0), wq_col.struct(), out.data_ptr(),
                                      out.stride(0), code, dr, dc, seed, offset, rht_signs, ws.data_ptr(), ws.numel(),
                                      _stream_ptr(stream)), stream)
    return out, dyq_row, (dyq_col if save_col else None)


def linear_wgrad(dyq_col: QTensor, xq_col: QTensor, *, out_dtype=torch.bfloat16, accumulate=False, out=None,
                 stream=None):
    """nvfp4_linear_wgrad: dW [N, K] = Q(H dY)^T Q(H X)."""
    lib = _lib.load()
    if out is None:
        out = (torch.zeros if accumulate else torch.empty)((dyq_col.rows, xq_col.rows), dtype=out_dtype,
                                                           device=dyq_col.codes.device)
    code = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _checked(lib.nvfp4_linear_wgrad(dyq_col.struct(), xq_col.struct(), out.data_ptr(), out.stride(0), code,
                                      int(accumulate), _stream_ptr(stream)), stream)
    return out


def newton_schulz_workspace(m, n, device=None):
    """A device buffer of nvfp4_newton_schulz_workspace_size(m, n) bytes (256-byte aligned)."""
    nbytes = _lib.load().nvfp4_newton_schulz_workspace_size(m, n)
    if nbytes == 0:
        raise NVFP4Error(_lib.NVFP4_ERR_UNSUPPORTED_SHAPE, "no Newton-Schulz workspace for %dx%d" % (m, n))
    return torch.empty(nbytes, dtype=torch.uint8, device=device if device is not None else "cuda")


def newton_schulz(g: torch.Tensor, iters: int, *, normalize=True, out: Optional[torch.Tensor] = None,
                  norm: Optional[torch.Tensor] = None, workspace=None, stream=None):
    """nvfp4_newton_schulz on a BF16 [m, n] CUDA tensor: returns (X, ||G||_F as a 1-float
    device tensor, or None without normalisation).  out may be g itself (in place).

    The cubic iteration multiplies a small singular value by about 1.5 per step, and
    after the Frobenius normalisation the smallest ones start near 1/sqrt(m) of the
    largest or below, so a few-thousand-row matrix takes about 12-16 steps."""
    lib = _lib.load()
    if g.dtype != torch.bfloat16 or not g.is_cuda or g.dim() != 2 or g.stride(1) != 1:
        raise ValueError("g must be a 2-D BF16 CUDA tensor with a contiguous last dimension")
    m, n = g.shape
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=g.device)
    if normalize and norm is None:
        norm = torch.empty(1, dtype=torch.float32, device=g.device)
    if workspace is None:
        workspace = newton_schulz_workspace(m, n, g.device)
    _checked(lib.nvfp4_newton_schulz(g.data_ptr(), m, n, g.stride(0), out.data_ptr(), out.stride(0), int(iters),
                                       int(normalize), _ptr(norm) if normalize else None, workspace.data_ptr(),
                                       workspace.numel(), _stream_ptr(stream)), stream)
    return out, (norm if normalize else None)


def _bf16_matrix(t, name):
    if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("%s must be a 2-D BF16 CUDA tensor with a contiguous last dimension" % name)


def lora_residual(w: torch.Tensor, l: torch.Tensor, r: torch.Tensor, out: Optional[torch.Tensor] = None,
                  stream=None):
    """nvfp4_lora_residual: W_res = BF16(W - L R) (FP32 accumulation over the rank, in order)."""
    lib = _lib.load()
    for t, nm in ((w, "w"), (l, "l"), (r, "r")):
        _bf16_matrix(t, nm)
    N, K = w.shape
    rank = l.shape[1]
    if out is None:
        out = torch.empty_like(w)
    _checked(lib.nvfp4_lora_residual(w.data_ptr(), N, K, w.stride(0), l.data_ptr(), l.stride(0), r.data_ptr(),
                                       r.stride(0), rank, out.data_ptr(), out.stride(0), _stream_ptr(stream)), stream)
    return out


def lowrank_project(a: torch.Tensor, b: torch.Tensor, *, b_trans=False, out: Optional[torch.Tensor] = None,
                    stream=None):
    """nvfp4_lowrank_project: U = BF16(A B^T), B [r, K] (or its transpose [K, r] with b_trans)."""
    lib = _lib.load()
    _bf16_matrix(a, "a")
    _bf16_matrix(b, "b")
    M, K = a.shape
    rank = b.shape[1] if b_trans else b.shape[0]
    if out is None:
        out = torch.empty((M, rank), dtype=torch.bfloat16, device=a.device)
    _checked(lib.nvfp4_lowrank_project(a.data_ptr(), M, K, a.stride(0), b.data_ptr(), b.stride(0), int(b_trans),
                                         rank, out.data_ptr(), out.stride(0), _stream_ptr(stream)), stream)
    return out


def lowrank_project_scaled(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor, *,
                           b_trans=False, out: Optional[torch.Tensor] = None, stream=None):
    """nvfp4_lowrank_project_scaled: U' = BF16(A B^T / g), g = fl32(scale_a * scale_b) (two
    1-float device tensors, e.g. the tensor scales of an NVFP4 GEMM's operands)."""
    lib = _lib.load()
    _bf16_matrix(a, "a")
    _bf16_matrix(b, "b")
    M, K = a.shape
    rank = b.shape[1] if b_trans else b.shape[0]
    if out is None:
        out = torch.empty((M, rank), dtype=torch.bfloat16, device=a.device)
    _checked(lib.nvfp4_lowrank_project_scaled(a.data_ptr(), M, K, a.stride(0), b.data_ptr(), b.stride(0),
                                                int(b_trans), rank, scale_a.data_ptr(), scale_b.data_ptr(),
                                                out.data_ptr(), out.stride(0), _stream_ptr(stream)), stream)
    return out


def gemm_lowrank(A: QTensor, B: QTensor, u: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
                 stream=None):
    """nvfp4_gemm_lowrank: BF16 C = g (A . B^T + U V^T), g = S_A S_B; u [M, r], v [N, r] BF16."""
    lib = _lib.load()
    _bf16_matrix(u, "u")
    _bf16_matrix(v, "v")
    if out is None:
        out = torch.empty((A.rows, B.rows), dtype=torch.bfloat16, device=A.codes.device)
    _checked(lib.nvfp4_gemm_lowrank(A.struct(), B.struct(), u.data_ptr(), u.stride(0), v.data_ptr(), v.stride(0),
                                      u.shape[1], out.data_ptr(), out.stride(0), _stream_ptr(stream)), stream)
    return out


def lowrank_expand_add(y: torch.Tensor, u: torch.Tensor, c: torch.Tensor, *, c_trans=False, stream=None):
    """nvfp4_lowrank_expand_add: Y <- BF16(Y + U C^T) in place, C [N, r] (or [r, N] with c_trans)."""
    lib = _lib.load()
    for t, nm in ((y, "y"), (u, "u"), (c, "c")):
        _bf16_matrix(t, nm)
    M, N = y.shape
    rank = u.shape[1]
    _checked(lib.nvfp4_lowrank_expand_add(y.data_ptr(), M, N, y.stride(0), u.data_ptr(), u.stride(0), c.data_ptr(),
                                            c.stride(0), int(c_trans), rank, _stream_ptr(stream)), stream)
    return y


def lora_linear_fwd(x: torch.Tensor, wq_res_row: QTensor, l: torch.Tensor, r: torch.Tensor, *, save_col=True,
                    rht_signs=0, out=None, u=None, xq_row=None, xq_col=None, stream=None):
    """nvfp4_lora_linear_fwd: Y = BF16(g (Q(X) Q(W_res)^T + U' L^T)), U' = BF16(X R^T / g),
    g = S_X S_W, in one GEMM; returns (Y, Xq_row, Xq_col or None).  l [N, r] and r [r, K]
    contiguous."""
    lib = _lib.load()
    for t, nm in ((x, "x"), (l, "l"), (r, "r")):
        _bf16_matrix(t, nm)
    M, K = x.shape
    N = wq_res_row.rows
    rank = l.shape[1]
    if l.shape != (N, rank) or r.shape != (rank, K) or not (l.is_contiguous() and r.is_contiguous()):
        raise ValueError("l must be a contiguous [N, r] and r a contiguous [r, K] BF16 matrix")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if u is None:
        u = torch.empty((M, rank), dtype=torch.bfloat16, device=x.device)
    if xq_row is None:
        xq_row = QTensor.empty(M, K, SCALE_MMA, x.device)
    if save_col and xq_col is None:
        xq_col = QTensor.empty(K, M, SCALE_MMA, x.device)
    ws = workspace(x.device, stream)
    xc = xq_col.struct() if save_col else None
    _checked(lib.nvfp4_lora_linear_fwd(x.data_ptr(), M, K, x.stride(0), wq_res_row.struct(), l.data_ptr(),
                                         r.data_ptr(), rank, out.data_ptr(), out.stride(0), xq_row.struct(), xc,
                                         rht_signs, u.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream)), stream)
    return out, xq_row, (xq_col if save_col else None)


def lora_linear_dgrad(dy: torch.Tensor, wq_res_col: QTensor, l: torch.Tensor, rt: torch.Tensor, *, seed, offset=0,
                      save_col=True, rht_signs=0, out=None, u=None, dyq_row=None, dyq_col=None, stream=None):
    """nvfp4_lora_linear_dgrad: dX = BF16(g (Q_sr(dY) Q(W_res) + U' R)), U' = BF16(dY L / g),
    g = S_dY S_W, in one GEMM; returns (dX, dYq_row, dYq_col or None).  l [N, r] and
    rt = R^T [K, r] contiguous."""
    lib = _lib.load()
    for t, nm in ((dy, "dy"), (l, "l"), (rt, "rt")):
        _bf16_matrix(t, nm)
    M, N = dy.shape
    K = wq_res_col.rows
    rank = l.shape[1]
    if l.shape != (N, rank) or rt.shape != (K, rank) or not (l.is_contiguous() and rt.is_contiguous()):
        raise ValueError("l must be a contiguous [N, r] and rt a contiguous [K, r] BF16 matrix")
    if out is None:
        out = torch.empty((M, K), dtype=torch.bfloat16, device=dy.device)
    if u is None:
        u = torch.empty((M, rank), dtype=torch.bfloat16, device=dy.device)
    if dyq_row is None:
        dyq_row = QTensor.empty(M, N, SCALE_MMA, dy.device)
    if save_col and dyq_col is None:
        dyq_col = QTensor.empty(N, M, SCALE_MMA, dy.device)
    ws = workspace(dy.device, stream)
    dc = dyq_col.struct() if save_col else None
    _checked(lib.nvfp4_lora_linear_dgrad(dy.data_ptr(), M, N, dy.stride(0), wq_res_col.struct(), l.data_ptr(),
                                           rt.data_ptr(), rank, out.data_ptr(), out.stride(0), dyq_row.struct(), dc,
                                           seed, offset, rht_signs, u.data_ptr(), ws.data_ptr(), ws.numel(),
                                           _stream_ptr(stream)), stream)
    return out, dyq_row, (dyq_col if save_col else None)


def check_conversions(n_sr=1 << 26, stream=None):
    """nvfp4_check_conversions: mismatch counts (E2M1 RNE, E4M3, E2M1 SR) of the hardware
    conversions against their definitions on the current device; all 0 when conforming."""
    lib = _lib.load()
    counts = torch.zeros(4, dtype=torch.int64, device="cuda")
    _checked(lib.nvfp4_check_conversions(counts.data_ptr(), n_sr, _stream_ptr(stream)), stream)
    return [int(v) for v in counts[:3].cpu().tolist()]


def get_status(stream=None):
    """nvfp4_get_status: synchronise the stream and raise on a recorded device-side error."""
    lib = _lib.load()
    _lib.check(lib.nvfp4_get_status(_stream_ptr(stream)))
