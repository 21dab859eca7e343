"""CPU-side checks of the C ABI: the library builds for sm_100a, loads without a
GPU, exports every function include/nvfp4.h declares, and rejects bad arguments
before touching the device."""

import ctypes
import os
import re

import pytest

from nvfp4_pretraining_linear_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_library_exports_every_declared_function(lib):
    declared = header_functions()
    assert {"nvfp4_quantize", "nvfp4_dequantize", "nvfp4_gemm", "nvfp4_linear_fwd", "nvfp4_linear_dgrad",
            "nvfp4_linear_wgrad"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared <= set(_lib.SIGNATURES), declared - set(_lib.SIGNATURES)


def test_struct_layouts_match_header():
    # sizes follow from the header's field order (x86-64 / aarch64 ABI)
    assert ctypes.sizeof(_lib.NVFP4Tensor) == 8 * 3 + 8 * 2 + 4 * 2
    assert ctypes.sizeof(_lib.QuantOpts) == 4 * 4 + 8 * 2 + 4 * 2 + 8 * 2


def test_sizes(lib):
    assert lib.nvfp4_version() >= 100
    assert lib.nvfp4_workspace_size() >= 12
    assert lib.nvfp4_scales_bytes(256, 256, _lib.SCALE_ROWMAJOR) == 256 * 16
    assert lib.nvfp4_scales_bytes(256, 256, _lib.SCALE_MMA) == 256 * 16
    assert lib.nvfp4_scales_bytes(200, 80, _lib.SCALE_MMA) == 256 * 8   # rows padded to 128, blocks to 4
    assert lib.nvfp4_scales_bytes(16, 32, _lib.SCALE_ROWMAJOR) == 32


def _tensor(rows, cols, layout=_lib.SCALE_MMA, ptr=0x10000):
    return _lib.NVFP4Tensor(ptr, ptr + 0x100000, ptr + 0x200000, rows, cols, layout, 0)


def test_quantize_argument_errors(lib):
    opts = _lib.QuantOpts()
    t = _tensor(32, 48)
    st = lib.nvfp4_quantize(0x1000, 32, 48, 48, None, ctypes.byref(t), None, 0x2000, 256, None)
    assert st == 1  # opts NULL
    st = lib.nvfp4_quantize(0x1000, 32, 40, 40, ctypes.byref(opts), ctypes.byref(_tensor(32, 40)), None, 0x2000, 256, None)
    assert st == 2  # cols % 16
    st = lib.nvfp4_quantize(0x1000, 32, 48, 48, ctypes.byref(opts), None, None, 0x2000, 256, None)
    assert st == 1  # no output
    st = lib.nvfp4_quantize(0x1008, 32, 48, 48, ctypes.byref(opts), ctypes.byref(t), None, 0x2000, 256, None)
    assert st == 3  # misaligned x
    bad = _lib.QuantOpts(1, 0, 0, 1, 0, 0, 0, 0, None, None)
    st = lib.nvfp4_quantize(0x1000, 32, 48, 48, ctypes.byref(bad), ctypes.byref(t), None, 0x2000, 256, None)
    assert st == 1  # 2D with SR
    big = _lib.QuantOpts(1, 0, 0, 0, 0, 1 << 32, 0, 0, None, None)
    st = lib.nvfp4_quantize(0x1000, 32, 48, 48, ctypes.byref(big), ctypes.byref(t), None, 0x2000, 256, None)
    assert st == 1  # offset >= 2^32
    col = _tensor(48, 24)
    st = lib.nvfp4_quantize(0x1000, 24, 48, 48, ctypes.byref(opts), None, ctypes.byref(col), 0x2000, 256, None)
    assert st == 2  # col layout needs rows % 16
    st = lib.nvfp4_quantize(0x1000, 32, 48, 48, ctypes.byref(opts), ctypes.byref(_tensor(32, 64)), None, 0x2000, 256, None)
    assert st == 1  # shape mismatch
    st = lib.nvfp4_quantize(0x1000, 32, 48, 48, ctypes.byref(opts), ctypes.byref(t), None, None, 0, None)
    assert st == 6  # no workspace
    msg = lib.nvfp4_last_error_string().decode()
    assert "workspace" in msg


def test_gemm_argument_errors(lib):
    a = _tensor(128, 64)
    b = _tensor(128, 128)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), 0x1000, 128, 0, 1.0, 0, None) == 1  # K mismatch
    a = _tensor(100, 64)
    b = _tensor(128, 64)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), 0x1000, 128, 0, 1.0, 0, None) == 2  # M % 128
    a = _tensor(128, 64, _lib.SCALE_ROWMAJOR)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), 0x1000, 128, 0, 1.0, 0, None) == 1  # layout
    a = _tensor(128, 64)
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), 0x1004, 128, 0, 1.0, 0, None) == 3  # misaligned C
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), 0x1000, 128, 7, 1.0, 0, None) == 1  # dtype
    assert lib.nvfp4_gemm(None, ctypes.byref(b), 0x1000, 128, 0, 1.0, 0, None) == 1


def test_dequantize_argument_errors(lib):
    q = _tensor(32, 48)
    assert lib.nvfp4_dequantize(ctypes.byref(q), None, 48, 1, None) == 1
    assert lib.nvfp4_dequantize(ctypes.byref(q), 0x1000, 40, 1, None) == 1
    assert lib.nvfp4_dequantize(ctypes.byref(q), 0x1008, 48, 1, None) == 3


def test_newton_schulz_workspace_and_argument_errors(lib):
    m, n = 256, 512
    need = lib.nvfp4_newton_schulz_workspace_size(m, n)
    parts = (m * n // 2 + m * n // 16) * 2 + m * m * 2 + m * m // 2 + m * m // 16      # X row+col, R, R row
    assert parts <= need <= parts + 16 * 256
    assert lib.nvfp4_newton_schulz_workspace_size(200, 512) == 0
    assert lib.nvfp4_newton_schulz_workspace_size(256, 0) == 0
    g, x, ws = 0x100000, 0x200000, 0x300000

    def call(*, g=g, m=m, n=n, ldg=n, x=x, ldx=n, iters=1, ws=ws, wsb=need, norm=None):
        return lib.nvfp4_newton_schulz(g, m, n, ldg, x, ldx, iters, 1, norm, ws, wsb, None)

    assert call(m=192) == 2                     # m % 128
    assert call(n=320) == 2                     # n % 128
    assert call(g=None) == 1
    assert call(iters=-1) == 1
    assert call(ldx=n - 8) == 1
    assert call(x=0x200008) == 3                # X not 16-byte aligned
    assert call(ldg=n + 4) == 3                 # row stride not 16 bytes
    assert call(x=g, ldx=n + 8) == 1            # in place with different strides
    assert call(norm=0x400002) == 3
    assert call(wsb=need - 1) == 6
    assert call(ws=0x300010) == 3               # workspace not 256-byte aligned
    assert "workspace" in lib.nvfp4_last_error_string().decode()


def test_lowrank_argument_errors(lib):
    a, b, u, y = 0x100000, 0x200000, 0x300000, 0x400000
    assert lib.nvfp4_lowrank_project(a, 128, 256, 256, b, 256, 0, 24, u, 24, None) == 2       # rank not 16k
    assert lib.nvfp4_lowrank_project(a, 128, 256, 256, b, 256, 0, 80, u, 80, None) == 2       # rank above 64
    assert lib.nvfp4_lowrank_project(a, 104, 256, 256, b, 256, 0, 32, u, 32, None) == 2       # M % 16
    assert lib.nvfp4_lowrank_project(a, 128, 200, 200, b, 200, 0, 32, u, 32, None) == 2       # K % 64
    assert lib.nvfp4_lowrank_project(a, 128, 256, 256, b, 16, 1, 32, u, 32, None) == 1        # ldb < rank (transposed)
    assert lib.nvfp4_lowrank_project(a + 8, 128, 256, 256, b, 256, 0, 32, u, 32, None) == 3
    assert lib.nvfp4_lowrank_project(None, 128, 256, 256, b, 256, 0, 32, u, 32, None) == 1
    assert lib.nvfp4_lowrank_expand_add(y, 128, 192, 192, u, 32, b, 32, 0, 32, None) == 2     # N % 128
    assert lib.nvfp4_lowrank_expand_add(y, 128, 256, 256, u, 32, b, 128, 1, 32, None) == 1    # ldc < N (transposed)
    assert lib.nvfp4_lowrank_expand_add(y, 128, 256, 260, u, 32, b, 32, 0, 32, None) == 3     # ldy % 8
    assert lib.nvfp4_lora_residual(y, 64, 100, 100, b, 32, a, 100, 32, u, 100, None) == 2     # K % 8
    assert lib.nvfp4_lora_residual(y, 64, 128, 128, b, 16, a, 128, 32, u, 128, None) == 1     # ldl < rank
    assert lib.nvfp4_lora_residual(y + 4, 64, 128, 128, b, 32, a, 128, 32, u, 128, None) == 3
    assert lib.nvfp4_lora_residual(y, 64, 128, 128, b, 32, a, 128, 8, u, 128, None) == 2       # rank 8


def test_lora_linear_checks_its_branch_before_launching(lib):
    """Every argument error of the composed LoRA-SVD calls returns before the NVFP4 part
    launches (no GPU here: reaching a launch would fail differently)."""
    w = _tensor(256, 384)
    x, l, r, u, y, ws = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000, 0x600000
    xr = _tensor(256, 384)

    def fwd(**kw):
        a = dict(x=x, m=256, k=384, ldx=384, w=ctypes.byref(w), l=l, r=r, rank=32, y=y, ldy=256,
                 xr=ctypes.byref(xr), u=u)
        a.update(kw)
        return lib.nvfp4_lora_linear_fwd(a["x"], a["m"], a["k"], a["ldx"], a["w"], a["l"], a["r"], a["rank"], a["y"],
                                         a["ldy"], a["xr"], None, 0, a["u"], ws, 256, None)

    assert fwd(rank=24) == 2
    assert fwd(u=None) == 1
    assert fwd(l=0x200008) == 3
    assert fwd(m=192) == 2                      # output rows % 128
    w352 = _tensor(256, 352)
    assert fwd(k=352, ldx=352, w=ctypes.byref(w352)) == 2     # inner % 64
    assert fwd(w=None) == 1
    assert lib.nvfp4_lora_linear_dgrad(y, 256, 256, 256, ctypes.byref(_tensor(384, 256)), l, r, 32, x, 384,
                                       ctypes.byref(_tensor(256, 256)), None, 1, 0, 0, None, ws, 256, None) == 1


def test_grouped_lowrank_and_scaled_projection_argument_errors(lib):
    """The grouped GEMM, the GEMM with a low-rank term and the scaled projection reject
    bad arguments before any launch."""
    T_P = ctypes.POINTER(_lib.NVFP4Tensor)
    a, b = _tensor(256, 512), _tensor(384, 512)
    arr_a = (T_P * 2)(ctypes.pointer(a), ctypes.pointer(a))
    arr_b = (T_P * 2)(ctypes.pointer(b), ctypes.pointer(b))
    arr_c = (ctypes.c_void_p * 2)(0x700000, 0x800000)
    arr_ld = (ctypes.c_int64 * 2)(384, 384)
    assert lib.nvfp4_gemm_grouped(arr_a, arr_b, arr_c, arr_ld, 0, 1, None) == 1          # count 0
    assert lib.nvfp4_gemm_grouped(arr_a, arr_b, arr_c, arr_ld, 9, 1, None) == 1          # count above 8
    assert lib.nvfp4_gemm_grouped(arr_a, arr_b, arr_c, arr_ld, 2, 7, None) == 1          # out_dtype
    assert lib.nvfp4_gemm_grouped(None, arr_b, arr_c, arr_ld, 2, 1, None) == 1
    bad_k = _tensor(384, 320)
    arr_b2 = (T_P * 2)(ctypes.pointer(b), ctypes.pointer(bad_k))
    assert lib.nvfp4_gemm_grouped(arr_a, arr_b2, arr_c, arr_ld, 2, 1, None) == 1         # A.cols != B.cols
    arr_ld2 = (ctypes.c_int64 * 2)(384, 100)
    assert lib.nvfp4_gemm_grouped(arr_a, arr_b, arr_c, arr_ld2, 2, 1, None) == 1         # ldc < N
    arr_c2 = (ctypes.c_void_p * 2)(0x700000, 0x800008)
    assert lib.nvfp4_gemm_grouped(arr_a, arr_b, arr_c2, arr_ld, 2, 1, None) == 3         # misaligned C
    u, v = 0x900000, 0xA00000
    assert lib.nvfp4_gemm_lowrank(ctypes.byref(a), ctypes.byref(b), u, 32, v, 32, 24, 0x700000, 384, None) == 2
    assert lib.nvfp4_gemm_lowrank(ctypes.byref(a), ctypes.byref(b), None, 32, v, 32, 32, 0x700000, 384, None) == 1
    assert lib.nvfp4_gemm_lowrank(ctypes.byref(a), ctypes.byref(b), u, 16, v, 32, 32, 0x700000, 384, None) == 1
    assert lib.nvfp4_gemm_lowrank(ctypes.byref(a), ctypes.byref(b), u + 8, 32, v, 32, 32, 0x700000, 384, None) == 3
    s = 0xB00000
    assert lib.nvfp4_lowrank_project_scaled(0x100000, 128, 256, 256, 0x200000, 256, 0, 32, None, s, u, 32,
                                            None) == 1
    assert lib.nvfp4_lowrank_project_scaled(0x100000, 128, 256, 256, 0x200000, 256, 0, 24, s, s, u, 24,
                                            None) == 2
