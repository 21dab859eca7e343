"""Failure detection on the GPU without a fault: host-side injection makes one
bounded device-side wait run out; the library must report NVFP4_ERR_TIMEOUT through
nvfp4_get_status, and the context must stay usable (exact results afterwards)."""

import pytest

from nvfp4_pretraining_linear_b200 import api, synthetic, _lib
from oracle import nvfp4_oracle as O
from tests.helpers import assert_layout_equal, bf16_to_np

pytestmark = pytest.mark.gpu


def test_skipped_tile_load_reports_timeout_and_context_survives(monkeypatch):
    x = synthetic.normal((1024, 1024), 1.0, seed=7, device="cuda")
    api.get_status()                                        # start from a clean status word
    monkeypatch.setenv("NVFP4_INJECT_SKIP_TILE", "5")       # tile 5 of 64 is never loaded
    api.quantize(x, emit_row=True, emit_col=True)
    with pytest.raises(_lib.NVFP4Error) as err:
        api.get_status()
    assert err.value.status == _lib.NVFP4_ERR_TIMEOUT
    api.get_status()                                        # the status word was cleared by the report
    monkeypatch.delenv("NVFP4_INJECT_SKIP_TILE")
    rq, cq = api.quantize(x, emit_row=True, emit_col=True)
    ref = O.quantize(bf16_to_np(x), emit_row=True, emit_col=True)
    assert_layout_equal(rq, ref["row"], "row after the injected timeout")
    assert_layout_equal(cq, ref["col"], "col after the injected timeout")
    api.get_status()


def test_gemm_skipped_stage_reports_timeout_and_context_survives(monkeypatch):
    """The same for the CTA-pair GEMM: with NVFP4_INJECT_GEMM_SKIP_STAGE=3 the first CTA
    pair never loads its fourth K-stage, so the MMA issuers' bounded wait runs out; every
    role of both CTAs winds down with bounded waits and frees its tensor memory, the
    library reports NVFP4_ERR_TIMEOUT, and the next GEMM is within the bound."""
    import torch

    from tests.helpers import gemm_check

    M, N, K = 512, 512, 2048                                 # 8 K-stages per tile, 4 tiles
    a = synthetic.normal((M, K), 1.0, seed=17, device="cuda")
    b = synthetic.normal((N, K), 1.0, seed=18, device="cuda")
    qa, _ = api.quantize(a)
    qb, _ = api.quantize(b)
    api.get_status()
    monkeypatch.setenv("NVFP4_INJECT_GEMM_SKIP_STAGE", "3")
    api.gemm(qa, qb, out_dtype=torch.float32)
    with pytest.raises(_lib.NVFP4Error) as err:
        api.get_status()
    assert err.value.status == _lib.NVFP4_ERR_TIMEOUT
    api.get_status()
    monkeypatch.delenv("NVFP4_INJECT_GEMM_SKIP_STAGE")
    c = api.gemm(qa, qb, out_dtype=torch.float32)
    api.get_status()
    ra = O.quantize(bf16_to_np(a))["row"]
    rb = O.quantize(bf16_to_np(b))["row"]
    assert gemm_check(c.cpu().numpy(), O.dequantize(*ra), O.dequantize(*rb)) <= 1.0
