"""The allocation-free quantiser entry point (nvfp4_quantize_noalloc), called
through the C ABI, gives the same bytes and maxima as nvfp4_quantize with a
caller workspace -- on two calls in a row, the second with a smaller tensor
maximum so that stale scratch from the first call would show up in the tensor
scales -- in each of the quantiser's families of modes: round-to-nearest row
layout only, 2D 16x16 weight blocks with both layouts, and stochastic rounding
with the Hadamard transform on both layouts.

This file is collected last on purpose: it needs nothing from the other tests
and passes alone in a fresh process as well as after them."""

import ctypes

import pytest
import torch

from nvfp4_pretraining_linear_b200 import _lib, api, synthetic

pytestmark = pytest.mark.gpu

MODES = {
    "rne_row": dict(emit_col=False),
    "2d_row_col": dict(block_2d=True),
    "sr_rht_both": dict(stochastic=True, rht_row=True, rht_col=True, seed=1234, offset=5, rht_signs=0x5A3C),
}


def _opts(kw, amax_out):
    return _lib.QuantOpts(int(kw.get("stochastic", False)), int(kw.get("rht_row", False)),
                          int(kw.get("rht_col", False)), int(kw.get("block_2d", False)), kw.get("seed", 0),
                          kw.get("offset", 0), kw.get("rht_signs", 0), 0, None, amax_out.data_ptr())


def _via_noalloc(lib, x, kw, emit_col):
    rows, cols = x.shape
    rq = api.QTensor.empty(rows, cols, api.SCALE_MMA, x.device)
    cq = api.QTensor.empty(cols, rows, api.SCALE_MMA, x.device) if emit_col else None
    amax = torch.full((3,), -1.0, dtype=torch.float32, device=x.device)
    opts = _opts(kw, amax)
    rs = rq.struct()
    cs = cq.struct() if emit_col else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.nvfp4_quantize_noalloc(x.data_ptr(), rows, cols, x.stride(0), ctypes.byref(opts), ctypes.byref(rs),
                                    ctypes.byref(cs) if emit_col else None, stream)
    assert st == 0, lib.nvfp4_last_error_string()
    return rq, cq, amax


def _same(a, b):
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert a.tensor_scale.view(torch.int32).item() == b.tensor_scale.view(torch.int32).item()


@pytest.mark.parametrize("mode", list(MODES))
def test_quantize_noalloc_matches_workspace_entry_point_twice(mode):
    lib = _lib.load()
    kw = dict(MODES[mode])
    emit_col = kw.pop("emit_col", True)
    first = synthetic.normal((384, 640), 1.0, seed=41, device="cuda", outlier_frac=0.01, outlier_mult=50.0)
    second = synthetic.normal((256, 512), 0.01, seed=42, device="cuda")       # far smaller maximum
    for x in (first, second):
        amax_ref = torch.full((3,), -1.0, dtype=torch.float32, device="cuda")
        rq_ref, cq_ref = api.quantize(x, emit_row=True, emit_col=emit_col, amax_out=amax_ref, **kw)
        rq, cq, amax = _via_noalloc(lib, x, kw, emit_col)
        _same(rq, rq_ref)
        if emit_col:
            _same(cq, cq_ref)
        assert torch.equal(amax.view(torch.int32), amax_ref.view(torch.int32))
    api.get_status()
