"""ctypes view of the C ABI in include/nvfp4.h (argument marshalling only)."""

import ctypes
import os
import threading

from . import build as _build

c_void_p = ctypes.c_void_p
c_int32 = ctypes.c_int32
c_int64 = ctypes.c_int64
c_uint32 = ctypes.c_uint32
c_uint64 = ctypes.c_uint64
c_size_t = ctypes.c_size_t
c_float = ctypes.c_float

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARG = 1
NVFP4_ERR_UNSUPPORTED_SHAPE = 2
NVFP4_ERR_MISALIGNED = 3
NVFP4_ERR_CUDA = 4
NVFP4_ERR_TIMEOUT = 5
NVFP4_ERR_WORKSPACE = 6
STATUS_NAMES = {
    0: "NVFP4_OK",
    1: "NVFP4_ERR_INVALID_ARG",
    2: "NVFP4_ERR_UNSUPPORTED_SHAPE",
    3: "NVFP4_ERR_MISALIGNED",
    4: "NVFP4_ERR_CUDA",
    5: "NVFP4_ERR_TIMEOUT",
    6: "NVFP4_ERR_WORKSPACE",
}
SCALE_ROWMAJOR = 0
SCALE_MMA = 1
OUT_BF16 = 0
OUT_F32 = 1


class NVFP4Tensor(ctypes.Structure):
    _fields_ = [
        ("codes", c_void_p),
        ("scales", c_void_p),
        ("tensor_scale", c_void_p),
        ("rows", c_int64),
        ("cols", c_int64),
        ("scale_layout", c_int32),
        ("reserved", c_int32),
    ]


class QuantOpts(ctypes.Structure):
    _fields_ = [
        ("stochastic", c_int32),
        ("rht_row", c_int32),
        ("rht_col", c_int32),
        ("block_2d", c_int32),
        ("seed", c_uint64),
        ("offset", c_uint64),
        ("rht_signs", c_uint32),
        ("reserved", c_uint32),
        ("amax_in", c_void_p),
        ("amax_out", c_void_p),
    ]


T_P = ctypes.POINTER(NVFP4Tensor)
O_P = ctypes.POINTER(QuantOpts)

# name -> (restype, argtypes); the exported surface of include/nvfp4.h
SIGNATURES = {
    "nvfp4_version": (ctypes.c_int, []),
    "nvfp4_workspace_size": (c_size_t, []),
    "nvfp4_scales_bytes": (c_size_t, [c_int64, c_int64, c_int32]),
    "nvfp4_quantize": (c_int32, [c_void_p, c_int64, c_int64, c_int64, O_P, T_P, T_P, c_void_p, c_size_t, c_void_p]),
    "nvfp4_dequantize": (c_int32, [T_P, c_void_p, c_int64, c_int32, c_void_p]),
    "nvfp4_gemm": (c_int32, [T_P, T_P, c_void_p, c_int64, c_int32, c_float, c_int32, c_void_p]),
    "nvfp4_gemm_amax": (c_int32, [T_P, T_P, c_void_p, c_int64, c_float, c_uint32, c_void_p, c_void_p]),
    "nvfp4_linear_fwd": (c_int32, [c_void_p, c_int64, c_int64, c_int64, T_P, c_void_p, c_int64, c_int32, T_P, T_P,
                                   c_uint32, c_void_p, c_size_t, c_void_p]),
    "nvfp4_linear_dgrad": (c_int32, [c_void_p, c_int64, c_int64, c_int64, T_P, c_void_p, c_int64, c_int32, T_P, T_P,
                                     c_uint64, c_uint64, c_uint32, c_void_p, c_size_t, c_void_p]),
    "nvfp4_linear_wgrad": (c_int32, [T_P, T_P, c_void_p, c_int64, c_int32, c_int32, c_void_p]),
    "nvfp4_newton_schulz_workspace_size": (c_size_t, [c_int64, c_int64]),
    "nvfp4_newton_schulz": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_int32, c_int32,
                                      c_void_p, c_void_p, c_size_t, c_void_p]),
    "nvfp4_lora_residual": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_void_p, c_int64,
                                      c_int32, c_void_p, c_int64, c_void_p]),
    "nvfp4_lowrank_project": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_int32, c_int32,
                                        c_void_p, c_int64, c_void_p]),
    "nvfp4_lowrank_project_scaled": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_int32,
                                                c_int32, c_void_p, c_void_p, c_void_p, c_int64, c_void_p]),
    "nvfp4_gemm_grouped": (c_int32, [ctypes.POINTER(T_P), ctypes.POINTER(T_P), ctypes.POINTER(c_void_p),
                                      ctypes.POINTER(c_int64), c_int32, c_int32, c_void_p]),
    "nvfp4_gemm_lowrank": (c_int32, [T_P, T_P, c_void_p, c_int64, c_void_p, c_int64, c_int32, c_void_p, c_int64,
                                      c_void_p]),
    "nvfp4_lowrank_expand_add": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_void_p, c_int64,
                                           c_int32, c_int32, c_void_p]),
    "nvfp4_lora_linear_fwd": (c_int32, [c_void_p, c_int64, c_int64, c_int64, T_P, c_void_p, c_void_p, c_int32,
                                        c_void_p, c_int64, T_P, T_P, c_uint32, c_void_p, c_void_p, c_size_t,
                                        c_void_p]),
    "nvfp4_lora_linear_dgrad": (c_int32, [c_void_p, c_int64, c_int64, c_int64, T_P, c_void_p, c_void_p, c_int32,
                                          c_void_p, c_int64, T_P, T_P, c_uint64, c_uint64, c_uint32, c_void_p,
                                          c_void_p, c_size_t, c_void_p]),
    "nvfp4_quantize_noalloc": (c_int32, [c_void_p, c_int64, c_int64, c_int64, O_P, T_P, T_P, c_void_p]),
    "nvfp4_check_conversions": (c_int32, [c_void_p, c_uint64, c_void_p]),
    "nvfp4_get_status": (c_int32, [c_void_p]),
    "nvfp4_last_error_string": (ctypes.c_char_p, []),
}

_lib = None
_lock = threading.Lock()


def lib_path():
    return _build.LIB_PATH


def load(build_if_missing=True):
    """Load libnvfp4.so (building it first if it is missing or stale).

    There is no fallback: a missing or unloadable library raises.
    """
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.LIB_PATH
        if build_if_missing and not _build.up_to_date():
            _build.build()
        if not os.path.exists(path):
            raise RuntimeError("libnvfp4.so is not built (run nvfp4_pretraining_linear_b200/build.py)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


class NVFP4Error(RuntimeError):
    def __init__(self, status, message):
        self.status = status
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, str(status)), message))


def check(status):
    if status != NVFP4_OK:
        msg = load().nvfp4_last_error_string()
        raise NVFP4Error(status, msg.decode() if msg else "")
    return status
