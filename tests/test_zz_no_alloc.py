"""The allocation-free quantiser entry point (nvfp4_quantize_noalloc), called
through the C ABI, gives the same bytes as nvfp4_quantize with a caller
workspace -- on two calls in a row, the second with a smaller tensor maximum so
that stale scratch from the first call would show up in the tensor scale.

This file is collected last on purpose: it needs nothing from the other tests
and passes alone in a fresh process as well as after them."""

import ctypes

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import _lib, api, synthetic

pytestmark = pytest.mark.gpu


def _via_noalloc(lib, x, opts_kw):
    rows, cols = x.shape
    rq = api.QTensor.empty(rows, cols, api.SCALE_MMA, x.device)
    cq = api.QTensor.empty(cols, rows, api.SCALE_MMA, x.device)
    o = opts_kw
    opts = _lib.QuantOpts(int(o["stochastic"]), 0, int(o["rht_col"]), 0, o["seed"], o["offset"], o["rht_signs"], 0,
                          None, None)
    rs, cs = rq.struct(), cq.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.nvfp4_quantize_noalloc(x.data_ptr(), rows, cols, x.stride(0), ctypes.byref(opts), ctypes.byref(rs),
                                    ctypes.byref(cs), stream)
    assert st == 0, lib.nvfp4_last_error_string()
    return rq, cq


def _same(a, b):
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert a.tensor_scale.view(torch.int32).item() == b.tensor_scale.view(torch.int32).item()


def test_quantize_noalloc_matches_workspace_entry_point_twice():
    lib = _lib.load()
    kw = dict(stochastic=True, rht_col=True, seed=1234, offset=5, rht_signs=0x5A3C)
    first = synthetic.normal((384, 640), 1.0, seed=41, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
    second = synthetic.normal((256, 512), 0.01, seed=42, device="cuda")       # far smaller maximum
    for x in (first, second):
        rq_ref, cq_ref = api.quantize(x, emit_row=True, emit_col=True, **kw)
        rq, cq = _via_noalloc(lib, x, kw)
        _same(rq, rq_ref)
        _same(cq, cq_ref)
    api.get_status()
