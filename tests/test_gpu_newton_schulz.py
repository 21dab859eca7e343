"""GPU parity of nvfp4_newton_schulz (the cubic Newton-Schulz iteration with NVFP4
products, residual form) against the oracle.

- Normalisation: X_0 and ||G||_F bit for bit.
- One step, exact construction: X from tests.helpers.exact_operand has tensor scale
  2^-9 and products whose partial sums are exact in FP32, so the residual
  R = BF16(I - X X^T) is predicted bit for bit (checked through nvfp4_gemm adding into
  I), its quantisation is then identical, and the new iterate must lie within the GEMM
  bound of the oracle's value before its BF16 rounding (the BF16 reading: bound +
  2^-8 |ref|).
- Many steps: quantisation decisions at rounding boundaries make trajectories drift
  apart (two oracle runs from inputs one BF16 ulp apart in 50 places end about 0.08
  apart per row after 12 steps), so the GPU is held to the properties the oracle itself
  meets: singular values near 1, distance to the SVD polar factor, and distance to the
  oracle's iterate.
"""

import numpy as np
import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic
from oracle import nvfp4_oracle as O
from tests.helpers import bf16_to_np, exact_operand

pytestmark = pytest.mark.gpu


def bits(x: torch.Tensor) -> np.ndarray:
    return x.view(torch.int16).cpu().numpy().astype(np.uint16)


def bits_t(x: torch.Tensor) -> torch.Tensor:
    return x.view(torch.int16)


def f32_bits(v) -> int:
    return int(np.float32(v).view(np.uint32))


@pytest.mark.parametrize("m,n", [(256, 512), (384, 1152)])
def test_normalisation_bit_exact(m, n):
    g = synthetic.student_t((m, n), 3, 0.1, seed=41 + m, device="cuda")
    x, nrm = api.newton_schulz(g, iters=0)
    want_x, want_n = O.ns_normalize(bf16_to_np(g))
    assert f32_bits(nrm.item()) == f32_bits(want_n)
    assert (bits(x) == O.f32_to_bf16_bits(want_x)).all()


def test_zero_input_and_copy_modes():
    g = torch.zeros((256, 384), dtype=torch.bfloat16, device="cuda")
    x, nrm = api.newton_schulz(g, iters=2)
    assert nrm.item() == 0.0 and not x.float().abs().max().item()
    h = synthetic.normal((256, 384), 1.0, seed=45, device="cuda")
    x, nrm = api.newton_schulz(h, iters=0, normalize=False)
    assert nrm is None and torch.equal(bits_t(x), bits_t(h))
    h2 = h.clone()
    api.newton_schulz(h2, iters=0, out=h2)                                # in-place normalisation
    want_x, _ = O.ns_normalize(bf16_to_np(h))
    assert (bits(h2) == O.f32_to_bf16_bits(want_x)).all()


@pytest.mark.parametrize("m,n", [(128, 256), (256, 512), (384, 768)])
def test_one_step_exact_construction(m, n):
    x, xv = exact_operand(m, n, seed=7 * m + n)
    assert (np.abs(xv).astype(np.float64) @ np.abs(xv).T.astype(np.float64)).max() < 8192  # FP32-exact sums
    want, parts = O.ns_step(xv)

    # the residual through the library's own GEMM adding into I: bit for bit
    xr, _ = api.quantize(x)
    r = torch.eye(m, dtype=torch.bfloat16, device="cuda")
    api.gemm(xr, xr, alpha=-1.0, accumulate=True, out=r)
    assert (bits(r) == O.f32_to_bf16_bits(parts["r"])).all()

    got, _ = api.newton_schulz(x, iters=1, normalize=False)
    api.get_status()
    # against the oracle's value before its own BF16 rounding (the BF16 reading: the GEMM
    # bound plus one BF16 half-ulp, 2^-8 |ref|); the rounded values may differ by an ulp
    pre = (O.gemm_ref(parts["r_hat"], parts["x_col"], 0.5).astype(np.float32) + xv).astype(np.float64)
    assert (O.bf16_round(pre.astype(np.float32)) == want).all()
    bound = 0.5 * O.gemm_tolerance(parts["r_hat"], parts["x_col"]) + 2.0 ** -8 * np.abs(pre)
    err = np.abs(bf16_to_np(got).astype(np.float64) - pre)
    assert (err <= bound).all(), float((err / bound).max())


@pytest.mark.parametrize("m,n,iters", [(256, 512, 12), (128, 384, 12)])
def test_iterations_converge_like_the_oracle(m, n, iters):
    g = synthetic.spectrum(m, n, 0.1, 1.0, seed=43 + m, device="cuda")
    x, nrm = api.newton_schulz(g, iters=iters)
    api.get_status()
    gv = bf16_to_np(g)
    want, want_n = O.newton_schulz(gv, iters)
    assert f32_bits(nrm.item()) == f32_bits(want_n)
    u, _, vt = np.linalg.svd(gv.astype(np.float64), full_matrices=False)
    polar = u @ vt
    xv = bf16_to_np(x).astype(np.float64)
    for name, v in (("gpu", xv), ("oracle", want.astype(np.float64))):
        sv = np.linalg.svd(v, compute_uv=False)
        assert 0.8 < sv.min() and sv.max() < 1.2, (name, sv.min(), sv.max())
        assert np.linalg.norm(v - polar) / np.sqrt(m) < 0.2, name
    assert np.linalg.norm(xv - want) / np.sqrt(m) < 0.15


def test_full_size_properties():
    """A 3072 x 8192 Gaussian matrix (the shape of the 3B model's down-projection
    update, wide orientation), 16 steps: finite, every singular value within 20 % of 1
    (eigenvalues of X X^T in FP64), the norm within FP32 rounding of the FP64 norm."""
    m, n = 3072, 8192
    g = synthetic.normal((m, n), 1.0, seed=44, device="cuda")
    x, nrm = api.newton_schulz(g, iters=16)
    api.get_status()
    want_n = torch.linalg.vector_norm(g.double()).item()
    assert abs(nrm.item() - want_n) <= 2.0 ** -23 * want_n
    xd = x.double()
    assert torch.isfinite(xd).all()
    ev = torch.linalg.eigvalsh(xd @ xd.T)
    sv = ev.clamp_min(0).sqrt()
    assert 0.8 < sv.min().item() and sv.max().item() < 1.2, (sv.min().item(), sv.max().item())


def test_rejects_bad_shapes():
    g = synthetic.normal((200, 256), 1.0, seed=1, device="cuda")
    with pytest.raises(api.NVFP4Error):
        api.newton_schulz(g, iters=1)
