"""Pins for the CPU oracle: each test checks the oracle against something other than
itself -- an independent library cast or routine, a hand-derived example, a closed form,
an invariant of the NVFP4 format, or brute force on tiny inputs."""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def all_finite_bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_bits_to_f32(bits)
    return vals[np.isfinite(vals)]


# ---------------------------------------------------------------- E2M1 elements


def test_e2m1_value_set():
    codes = np.arange(16, dtype=np.uint8)
    vals = O.e2m1_decode(codes)
    assert sorted(set(np.abs(vals).tolist())) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.all(vals[8:] == -vals[:8])
    assert np.signbit(vals[8])  # code 0x8 is negative zero


def test_e2m1_rne_matches_ml_dtypes_on_every_bf16_value():
    """Library pin: ml_dtypes' float4_e2m1fn cast (round to nearest even, saturating)."""
    import ml_dtypes
    v = all_finite_bf16_values()
    ours = O.e2m1_encode_rne(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, ref)


def test_e2m1_rne_midpoints_and_saturation():
    import ml_dtypes
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=F32)
    eps = np.array([-1e-6, 0.0, 1e-6], dtype=F32)
    y = (mids[:, None] + eps[None, :] * mids[:, None]).reshape(-1)
    y = np.concatenate([y, -y, np.array([6.0, 6.5, 1e30, -7.0], F32)])
    ref = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(O.e2m1_encode_rne(y), ref)
    # hand table of the ties: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4
    assert O.e2m1_encode_rne(mids).tolist() == [0, 2, 2, 4, 4, 6, 6]


# ---------------------------------------------------------------- E4M3 scales


def test_e4m3_matches_torch_cast_on_bf16_grid_and_random():
    """Library pin: torch.float8_e4m3fn CPU cast (round to nearest even) after clamping to 448."""
    v = all_finite_bf16_values()
    v = v[~np.signbit(v)]  # block scales come from absolute maxima: never -0
    rng = np.random.default_rng(7)
    extra = np.concatenate([
        rng.uniform(0, 500, 200000).astype(F32),
        (2.0 ** rng.uniform(-14, 9.5, 200000)).astype(F32),
        np.array([0.0, 2 ** -10, 3 * 2 ** -11, 2 ** -9, 2 ** -6, 448.0, 464.0, 480.0, 1e30], F32),
    ])
    v = np.concatenate([v, extra]).astype(F32)
    clamped = np.minimum(v, F32(448.0))
    ref = torch.from_numpy(clamped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v), ref)


def test_e4m3_decode_matches_torch():
    b = np.arange(0x7F, dtype=np.uint8)  # every non-negative, non-NaN byte
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(O.e4m3_decode(b), ref)


def test_e4m3_matches_ml_dtypes():
    import ml_dtypes
    v = all_finite_bf16_values()
    v = np.minimum(v[~np.signbit(v)], F32(448.0))
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(O.e4m3_encode(v), ref)


# ---------------------------------------------------------------- bf16 helpers


def test_bf16_round_trip_matches_torch():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(100000) * 10 ** rng.uniform(-30, 30, 100000)).astype(F32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.f32_to_bf16_bits(x), ref)
    assert np.array_equal(O.bf16_bits_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


# ---------------------------------------------------------------- Philox4x32-10


def test_philox_known_answer_zero_key():
    # Philox4x32-10 with counter 0 and key 0: the generator's published known answer
    # (Salmon et al., SC'11 reference implementation), also what triton's Philox gives.
    w = O.philox4x32_10(0, 0, 0, 0, 0, 0)
    assert [int(v) for v in w] == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]


_TRITON_PHILOX = textwrap.dedent(r"""
    import os, sys, json
    os.environ["TRITON_INTERPRET"] = "1"
    import numpy as np, torch, triton, triton.language as tl

    @triton.jit
    def k(out_ptr, c_ptr, seed, n: tl.constexpr):
        offs = tl.arange(0, n)
        c0 = tl.load(c_ptr + offs * 4 + 0)
        c1 = tl.load(c_ptr + offs * 4 + 1)
        c2 = tl.load(c_ptr + offs * 4 + 2)
        c3 = tl.load(c_ptr + offs * 4 + 3)
        a, b, c, d = tl.philox(seed, c0, c1, c2, c3, n_rounds=10)
        tl.store(out_ptr + offs * 4 + 0, a)
        tl.store(out_ptr + offs * 4 + 1, b)
        tl.store(out_ptr + offs * 4 + 2, c)
        tl.store(out_ptr + offs * 4 + 3, d)

    cfg = json.loads(sys.argv[1])
    ctr = np.array(cfg["ctr"], dtype=np.uint32).reshape(-1, 4)
    out = torch.zeros(ctr.size, dtype=torch.int32)
    k[(1,)](out, torch.from_numpy(ctr.view(np.int32).reshape(-1).copy()), cfg["seed"], n=ctr.shape[0])
    print(json.dumps([int(v) & 0xFFFFFFFF for v in out.tolist()]))
""")


def test_philox_matches_triton_interpreter():
    """Library pin: triton.language.philox (4x32, 10 rounds) run by triton's CPU interpreter."""
    import json
    rng = np.random.default_rng(11)
    ctr = rng.integers(0, 2 ** 32, size=(64, 4), dtype=np.uint64)
    ctr[0] = 0
    ctr[1] = [5, 0, 1, 1234]
    ctr[2] = [0xFFFFFFFF] * 4
    for seed in (0, 1234, 0x0123456789ABCDEF, 2 ** 64 - 1):
        cfg = {"ctr": ctr.reshape(-1).tolist(), "seed": seed}
        env = dict(os.environ, TRITON_INTERPRET="1", CUDA_VISIBLE_DEVICES="")
        res = subprocess.run([sys.executable, "-c", _TRITON_PHILOX, json.dumps(cfg)], capture_output=True,
                             text=True, env=env, timeout=600)
        assert res.returncode == 0, res.stderr[-2000:]
        ref = np.array(json.loads(res.stdout.strip().splitlines()[-1]), dtype=np.uint64).reshape(-1, 4)
        ours = np.stack(O.philox4x32_10(ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3],
                                        seed & 0xFFFFFFFF, seed >> 32), axis=-1).astype(np.uint64)
        assert np.array_equal(ours, ref), seed


def test_philox_noise_uniform_and_stream_separation():
    n = O.philox_noise(0, 1 << 20, seed=1234, offset=0, tag=0)
    assert n.min() >= 0 and n.max() < 65536
    counts = np.bincount((n >> 8).astype(np.int64), minlength=256)
    exp = n.size / 256
    chi2 = ((counts - exp) ** 2 / exp).sum()
    assert chi2 < 350  # 255 dof: p ~ 1e-4 tail
    # tags and offsets give different streams
    n1 = O.philox_noise(0, 4096, seed=1234, offset=0, tag=1)
    n2 = O.philox_noise(0, 4096, seed=1234, offset=1, tag=0)
    assert not np.array_equal(n[:4096], n1) and not np.array_equal(n[:4096], n2)


def test_group_noise_mapping_by_hand():
    # w = 0x12345678: bytes (low..high) 0x78 0x56 0x34 0x12
    # n(e0) = 0x34*256 + 0x78 = 0x3478, n(e2) = 0x12*256 + 0x56 = 0x1256
    # bit-reversed over 16 bits: 0011010001111000 -> 0001111000101100 = 0x1E2C,
    #                            0001001001010110 -> 0110101001001000 = 0x6A48
    assert O.group_noise(np.array([0x12345678])).tolist() == [[0x3478, 0x1E2C, 0x1256, 0x6A48]]
    assert O.bitrev16(np.array([1, 0x00FF, 0x8000])).tolist() == [0x8000, 0xFF00, 1]
    # the word of group g is word g % 4 of Philox call g / 4
    w = O.philox4x32_10(3, 0, 1, 9, 77, 0)
    n = O.philox_noise(48, 16, seed=77, offset=9, tag=1)
    assert np.array_equal(n.reshape(4, 4), O.group_noise(np.array([int(v) for v in w])))


# ---------------------------------------------------------------- stochastic rounding


def test_sr_exact_count_over_all_noise():
    """Closed form: over every 16-bit n, the number of round-ups is floor(f * 2**16)."""
    rng = np.random.default_rng(5)
    ys = np.concatenate([rng.uniform(0, 6, 40), rng.uniform(0.5, 1, 10), rng.uniform(0, 0.01, 5),
                         np.array([0.3, 1.1, 2.9, 5.999, 1.0 + 2.0 ** -20, 0.25])]).astype(F32)
    nvals = np.arange(1 << 16)
    grid = O.E2M1_MAGNITUDES
    for y in ys:
        codes = O.e2m1_encode_sr(np.full(nvals.shape, y, F32), nvals)
        lo_i = np.searchsorted(grid, float(y), side="right") - 1
        f = (float(y) - grid[lo_i]) / (grid[lo_i + 1] - grid[lo_i])
        ups = int(np.count_nonzero(codes == lo_i + 1))
        assert ups == int(np.floor(f * 2 ** 16)), (y, ups)
        assert np.all((codes == lo_i) | (codes == lo_i + 1))


def test_sr_unbiased_statistically():
    rng = np.random.default_rng(9)
    ys = np.concatenate([rng.uniform(-6, 6, 30), np.array([0.1, -0.3, 5.5, -2.25])]).astype(F32)
    n = 1 << 18
    for j, y in enumerate(ys):
        noise = O.philox_noise(0, n, seed=99 + j, offset=j, tag=0)
        q = O.e2m1_decode(O.e2m1_encode_sr(np.full(n, y, F32), noise)).astype(np.float64)
        sd = q.std() + 1e-12
        # 16-bit noise: bias below 2**-16 of a grid step (<= 2)
        assert abs(q.mean() - float(y)) < 5 * sd / np.sqrt(n) + 2.0 * 2 ** -16, y


def test_sr_saturates_and_keeps_grid():
    noise = O.philox_noise(0, 1024, seed=1, offset=0, tag=0)
    assert np.all(O.e2m1_encode_sr(np.full(1024, 7.5, F32), noise) == 7)
    assert np.all(O.e2m1_encode_sr(np.full(1024, -6.0, F32), noise) == 15)
    assert np.all(O.e2m1_encode_sr(np.full(1024, 3.0, F32), noise) == 5)
    assert np.all(O.e2m1_encode_sr(np.full(1024, -0.0, F32), noise) == 8)


# ---------------------------------------------------------------- Hadamard


def test_rht_is_signed_sylvester_hadamard_over_four():
    """Library pin: scipy.linalg.hadamard(16) (Sylvester order); (H D / 4)(H D / 4)^T = I."""
    import scipy.linalg
    H = scipy.linalg.hadamard(16).astype(np.float64)
    for signs in (0x0000, 0xA5C3, 0xFFFF, 0x0001):
        D = np.diag([-1.0 if (signs >> j) & 1 else 1.0 for j in range(16)])
        cols = O.rht16(np.eye(16, dtype=F32), signs).astype(np.float64)  # row j = transform of e_j
        M = cols.T
        assert np.array_equal(M, H @ D / 4.0)
        assert np.array_equal(M @ M.T, np.eye(16))


def test_rht_preserves_wgrad_product_fp64():
    rng = np.random.default_rng(2)
    dy = rng.standard_normal((64, 24)).astype(F32)
    x = rng.standard_normal((64, 40)).astype(F32)
    t_dy = O.rht16(dy.T.reshape(24, 4, 16), 0x3C5A).reshape(24, 64).astype(np.float64)
    t_x = O.rht16(x.T.reshape(40, 4, 16), 0x3C5A).reshape(40, 64).astype(np.float64)
    ref = dy.T.astype(np.float64) @ x.astype(np.float64)
    np.testing.assert_allclose(t_dy @ t_x.T, ref, rtol=1e-5, atol=1e-4)


# ---------------------------------------------------------------- block / tensor scales


def test_hand_derived_block():
    spec = {}
    with open(os.path.join(GOLDEN, "hand_block.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            k, v = line.split(":", 1)
            spec[k.strip()] = v.split()
    x = np.array([float(t) for t in spec["x"]], F32).reshape(1, 16)
    q = O.quantize(x, emit_row=True)
    packed, scales, S = q["row"]
    assert F32(S).view(np.uint32) == int(spec["tensor_scale_bits"][0], 16)
    assert scales.tolist() == [[int(spec["scale_byte"][0], 16)]]
    assert O.unpack_codes(packed).reshape(-1).tolist() == [int(t) for t in spec["codes"]]
    assert packed.reshape(-1).tolist() == [int(t, 16) for t in spec["packed"]]


def _rand_tensor(rng, R, C, outliers=True):
    x = rng.standard_normal((R, C)).astype(F32)
    if outliers:
        m = rng.random((R, C)) < 0.01
        x[m] *= 50
    return O.bf16_bits_to_f32(O.f32_to_bf16_bits(x))


def test_block_absmax_lands_on_six_under_rne():
    """Format invariant: the block maximum (1 in 16 = 6.25 %) is coded +-6 when the
    block scale is a normal E4M3 number."""
    rng = np.random.default_rng(0)
    x = _rand_tensor(rng, 64, 256)
    for kw in ({}, {"block_2d": True}):
        q = O.quantize(x, emit_row=True, **kw)
        packed, scales, S = q["row"]
        codes = O.unpack_codes(packed).reshape(64, 16, 16)
        normal = scales >= 8
        vals = x.reshape(64, 16, 16)
        am = np.abs(vals).argmax(axis=-1)
        c_at_max = np.take_along_axis(codes, am[..., None], -1)[..., 0]
        if kw:
            # 2D: only the tile maximum itself is guaranteed to be +-6
            tile = np.abs(x).reshape(4, 16, 16, 16).max(axis=(1, 3))
            rowmax = np.abs(vals).max(axis=-1)
            is_tile_max = rowmax == np.repeat(tile, 16, axis=0)
            sel = normal & is_tile_max
        else:
            sel = normal
        assert sel.sum() > 10
        assert np.all((c_at_max[sel] & 7) == 7)


def test_power_of_two_scale_invariance():
    rng = np.random.default_rng(4)
    x = _rand_tensor(rng, 32, 128)
    q0 = O.quantize(x, emit_row=True, emit_col=True)
    for k in (-3, 5):
        qk = O.quantize((x * F32(2.0 ** k)).astype(F32), emit_row=True, emit_col=True)
        for lay in ("row", "col"):
            assert np.array_equal(q0[lay][0], qk[lay][0])
            assert np.array_equal(q0[lay][1], qk[lay][1])
            assert F32(qk[lay][2]) == F32(q0[lay][2] * F32(2.0 ** k))


def test_on_grid_round_trip_is_exact():
    rng = np.random.default_rng(6)
    R, C = 32, 64
    S = F32(2.0 ** -4)
    # block scales: powers of two; one block at 448 so the tensor amax is 6*448*S
    s_exp = rng.integers(-6, 8, size=(R, C // 16))
    s_val = (2.0 ** s_exp).astype(F32)
    s_val[0, 0] = 448.0
    idx = rng.integers(0, 8, size=(R, C))
    sign = rng.random((R, C)) < 0.5
    mag = O.E2M1_MAGNITUDES[idx]
    mag.reshape(R, C // 16, 16)[:, :, 0] = 6.0          # every block holds its maximum 6
    vals = np.where(sign, -mag, mag).reshape(R, C // 16, 16) * s_val[..., None] * float(S)
    x = vals.reshape(R, C).astype(F32)
    q = O.quantize(x, emit_row=True)
    packed, scales, S_q = q["row"]
    assert F32(S_q) == S
    assert np.array_equal(O.dequantize(packed, scales, S_q), x)


def test_2d_col_layout_is_transpose_of_row_layout():
    rng = np.random.default_rng(8)
    w = (rng.standard_normal((48, 80)) * 0.02).astype(F32)
    q = O.quantize_weight(w)
    r_codes = O.unpack_codes(q["row"][0])
    c_codes = O.unpack_codes(q["col"][0])
    assert np.array_equal(r_codes.T, c_codes)
    assert np.array_equal(O.dequantize(*q["row"]).T, O.dequantize(*q["col"]))
    # one scale per 16x16 tile
    s = q["row"][1]
    assert np.all(s.reshape(3, 16, 5) == s.reshape(3, 16, 5)[:, :1, :])


def test_zero_and_tiny_tensors():
    z = np.zeros((16, 32), F32)
    q = O.quantize(z, emit_row=True, emit_col=True)
    assert F32(q["row"][2]) == 1.0 and not q["row"][0].any() and not q["row"][1].any()
    # smallest BF16 subnormal amax: S is a tiny FP32 subnormal, block scales saturate or vanish
    t = np.zeros((16, 32), F32)
    t[3, 7] = O.bf16_bits_to_f32(np.array([1], np.uint16))[0]
    q = O.quantize(t, emit_row=True)
    assert q["row"][2] > 0
    deq = O.dequantize(*q["row"])
    assert np.all(np.isfinite(deq))


def test_rht_amax_sets_col_scale():
    rng = np.random.default_rng(12)
    x = _rand_tensor(rng, 32, 48)
    q = O.quantize(x, emit_row=True, emit_col=True, rht_col=True, rht_signs=0x1234)
    raw, rht_amax, _ = q["amax"]
    t = O.rht16(x.T.reshape(48, 2, 16), 0x1234)
    assert rht_amax == F32(np.abs(t).max())
    assert F32(q["col"][2]) == F32(rht_amax / F32(2688.0))
    assert F32(q["row"][2]) == F32(raw / F32(2688.0))


def test_nibble_order_low_is_even():
    assert O.pack_codes(np.array([[1, 2, 0xF, 0]], np.uint8)).tolist() == [[0x21, 0x0F]]


# ---------------------------------------------------------------- GEMM


def test_gemm_ref_brute_force():
    rng = np.random.default_rng(1)
    a = _rand_tensor(rng, 16, 32)
    b = _rand_tensor(rng, 16, 32)
    qa, qb = O.quantize(a)["row"], O.quantize(b)["row"]
    ah, bh = O.dequantize(*qa), O.dequantize(*qb)
    ref = O.gemm_ref(ah, bh, alpha=0.5)
    for m in range(16):
        for n in range(16):
            s = 0.0
            for k in range(32):
                s += float(ah[m, k]) * float(bh[n, k])
            assert abs(ref[m, n] - 0.5 * s) <= 1e-12 * (1 + abs(s))


def test_dequantize_brute_force():
    rng = np.random.default_rng(13)
    x = _rand_tensor(rng, 16, 32)
    packed, scales, S = O.quantize(x)["row"]
    deq = O.dequantize(packed, scales, S)
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for r in range(16):
        for c in range(32):
            byte = int(packed[r, c // 2])
            code = (byte >> 4) if c % 2 else (byte & 0xF)
            v = grid[code & 7] * (-1 if code & 8 else 1)
            sb = int(scales[r, c // 16])
            e, m = sb >> 3, sb & 7
            sv = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
            assert deq[r, c] == F32(F32(v * sv) * F32(S))


def test_linear_layer_refs_compose():
    rng = np.random.default_rng(21)
    M, K, N = 64, 48, 32
    x = _rand_tensor(rng, M, K)
    w = (rng.standard_normal((N, K)) * 0.02).astype(F32)
    dy = (rng.standard_normal((M, N)) * 1e-3).astype(F32)
    wq = O.quantize_weight(w)
    y, (ah, bh), xq = O.linear_fwd_ref(x, wq, rht_signs=0x00F0)
    assert y.shape == (M, N)
    # quantisation error is a few per cent of the unquantised product
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(y - exact) < 0.2 * np.linalg.norm(exact)
    dx, _, dyq = O.linear_dgrad_ref(dy, wq, seed=1234, offset=0, rht_signs=0x00F0)
    assert dx.shape == (M, K)
    exact = dy.astype(np.float64) @ w.astype(np.float64)
    assert np.linalg.norm(dx - exact) < 0.3 * np.linalg.norm(exact)
    dw, _ = O.linear_wgrad_ref(dyq, xq)
    exact = dy.T.astype(np.float64) @ x.astype(np.float64)
    assert dw.shape == (N, K)
    assert np.linalg.norm(dw - exact) < 0.3 * np.linalg.norm(exact)


# ---------------------------------------------------------------- recipe selection of the linear layer


def _hadamard_tokens(v, signs):
    """(1/4) H16 D applied to every 16-group along the last axis, from scipy's Sylvester
    Hadamard matrix in FP64 (independent of the oracle's butterfly)."""
    from scipy.linalg import hadamard
    d = np.array([-1.0 if (signs >> j) & 1 else 1.0 for j in range(16)])
    h = hadamard(16).astype(np.float64) / 4.0
    g = np.asarray(v, dtype=np.float64).reshape(v.shape[0], -1, 16) * d
    return (g @ h.T).reshape(v.shape)


def _grid_neighbours(layout):
    """Per element of a layout: its decoded value, and the magnitudes of the two grid
    points around y = x / (s S) for the value x it encodes (from ml_dtypes' float4 cast)."""
    import ml_dtypes
    packed, scales, S = layout
    codes = O.unpack_codes(packed)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mag = grid[codes & 7]
    sv = np.repeat(O.e4m3_decode(scales).astype(np.float64), 16, axis=1)
    return mag, sv, np.float64(S), ml_dtypes


def _rel(a, b):
    return np.linalg.norm(np.asarray(a, np.float64) - np.asarray(b, np.float64)) / np.linalg.norm(b)


def test_linear_recipe_selection():
    """Which operand gets which treatment in linear_fwd_ref / linear_dgrad_ref /
    linear_wgrad_ref, against what the recipe passage of the 12B NVFP4 page fixes:
    round-to-nearest for activations and weights, stochastic rounding for gradients
    only, the 16x16 Hadamard transform on both wgrad operands along the tokens (so it
    cancels in dY^T X), one 2D-quantised weight reused transposed by dgrad."""
    import ml_dtypes
    rng = np.random.default_rng(33)
    M, K, N, signs = 64, 48, 32, 0x5A3C
    x = _rand_tensor(rng, M, K)
    x[5, 7] = F32(80.0)                                    # an outlier that the transform spreads
    w = (rng.standard_normal((N, K)) * 0.02).astype(F32)
    dy = (rng.standard_normal((M, N)) * 1e-3).astype(F32)
    dy[9, 3] = F32(0.05)
    wq = O.quantize_weight(w)
    y, (xa, wb), xq = O.linear_fwd_ref(x, wq, rht_signs=signs)
    dx, (da, wcol), dyq = O.linear_dgrad_ref(dy, wq, seed=1234, offset=0, rht_signs=signs)
    dw, (ga, gb) = O.linear_wgrad_ref(dyq, xq)

    # fprop reads X's and W's row layouts; dgrad dY's row layout and W's exact transpose
    assert _rel(xa, x) < 0.1 and _rel(wb, w) < 0.2
    assert _rel(da, dy) < 0.15
    assert np.array_equal(wcol, wb.T)
    wr_codes, wc_codes = O.unpack_codes(wq["row"][0]), O.unpack_codes(wq["col"][0])
    assert np.array_equal(wc_codes, wr_codes.T)
    assert np.array_equal(wq["col"][1], np.repeat(wq["row"][1][::16, :].T, 16, axis=0))

    # wgrad reads both col layouts, each transformed along the tokens with the same signs
    assert _rel(ga, _hadamard_tokens(dy.T, signs)) < 0.15
    assert _rel(gb, _hadamard_tokens(x.T, signs)) < 0.1
    assert _rel(ga, dy.T) > 0.5 and _rel(gb, x.T) > 0.5
    assert _rel(dw, dy.T.astype(np.float64) @ x.astype(np.float64)) < 0.3

    # the col layouts' tensor scales come from the transformed maxima
    for q, v in ((xq, x), (dyq, dy)):
        t_amax = np.abs(_hadamard_tokens(v.T, signs)).max()
        assert abs(float(q["col"][2]) * 2688.0 / t_amax - 1.0) < 1e-6
        assert abs(float(q["row"][2]) * 2688.0 / np.abs(v).max() - 1.0) < 1e-6

    # round-to-nearest on X (both layouts) and W: each code is ml_dtypes' RNE cast of
    # y = x / (s S) -- the activation codes do not depend on any seed
    def rne_codes_match(layout, vals):
        packed, scales, S = layout
        sv = np.repeat(O.e4m3_decode(scales).astype(np.float32), 16, axis=1)
        d = (sv * F32(S)).astype(F32)
        r = np.where(d > 0, (F32(1.0) / np.where(d > 0, d, F32(1.0))).astype(F32), F32(0.0))
        yv = (vals * r).astype(F32)
        want = np.abs(np.clip(yv, -6, 6).astype(ml_dtypes.float4_e2m1fn).astype(np.float64))
        got = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])[O.unpack_codes(packed) & 7]
        return np.array_equal(got, want)

    assert rne_codes_match(xq["row"], x)
    assert rne_codes_match(xq["col"], _hadamard_tokens(x.T, signs).astype(F32)) or \
        rne_codes_match(xq["col"], O.rht16(x.T.reshape(K, -1, 16), signs).reshape(K, M))
    assert rne_codes_match(wq["row"], w)

    # stochastic rounding on dY only: its codes change with the seed (both layouts),
    # and some are not the nearest grid point
    _, _, dyq2 = O.linear_dgrad_ref(dy, wq, seed=4321, offset=0, rht_signs=signs)
    assert not np.array_equal(dyq["row"][0], dyq2["row"][0])
    assert not np.array_equal(dyq["col"][0], dyq2["col"][0])
    assert not rne_codes_match(dyq["row"], dy)
