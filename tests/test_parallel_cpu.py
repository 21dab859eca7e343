"""Data-parallel plumbing on CPU: world_size-2 gloo ranks exercise the token
sharding, per-rank SR offsets and the FP32 weight-gradient all-reduce (started
asynchronously per linear, waited once), with the oracle standing in for the
per-rank compute."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

F32 = np.float32

from nvfp4_pretraining_linear_b200.parallel import GradReducer, allreduce_grads, shard_tokens, sr_offset


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from oracle import nvfp4_oracle as O
    rng = np.random.default_rng(0)
    M, K, N = 256, 64, 48
    x = rng.standard_normal((M, K)).astype(np.float32)
    dy = (rng.standard_normal((M, N)) * 1e-3).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    lo, hi = shard_tokens(M, rank, world)
    wq = O.quantize_weight(w)
    _, _, xq = O.linear_fwd_ref(x[lo:hi], wq, rht_signs=0x1111)
    _, _, dyq = O.linear_dgrad_ref(dy[lo:hi], wq, seed=7, offset=sr_offset(3, rank, world), rht_signs=0x1111)
    dw, _ = O.linear_wgrad_ref(dyq, xq)
    g = torch.from_numpy(dw.astype(np.float32))
    np.save(os.path.join(out_dir, "partial%d.npy" % rank), g.numpy().copy())
    # two "linears": the second gradient's all-reduce starts before the first is waited on
    g2 = (g * 0.5).contiguous()
    red = GradReducer()
    red.start(g)
    red.start(g2)
    red.wait()
    np.save(os.path.join(out_dir, "dw%d.npy" % rank), g.numpy())
    np.save(os.path.join(out_dir, "dw2_%d.npy" % rank), g2.numpy())
    with pytest.raises(TypeError):
        allreduce_grads([g.to(torch.bfloat16)])
    # the per-rank dY layouts use distinct random words
    np.save(os.path.join(out_dir, "codes%d.npy" % rank), dyq["row"][0])
    dist.destroy_process_group()


def test_dp_wgrad_allreduce_gloo(tmp_path):
    world = 2
    port = _free_port()
    mp.spawn(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    d0 = np.load(tmp_path / "dw0.npy")
    d1 = np.load(tmp_path / "dw1.npy")
    assert np.array_equal(d0, d1)          # every rank holds the summed gradient
    p0, p1 = np.load(tmp_path / "partial0.npy"), np.load(tmp_path / "partial1.npy")
    assert d0.dtype == np.float32
    assert np.array_equal(d0, p0 + p1)     # the FP32 sum of the two FP32 partials, bit for bit
    assert np.array_equal(np.load(tmp_path / "dw2_0.npy"), (p0 * F32(0.5)) + (p1 * F32(0.5)))
    # the sum of the two shards' NVFP4 wgrads is close to the full unquantised dY^T X
    rng = np.random.default_rng(0)
    M, K, N = 256, 64, 48
    x = rng.standard_normal((M, K)).astype(np.float32)
    dy = (rng.standard_normal((M, N)) * 1e-3).astype(np.float32)
    exact = dy.T.astype(np.float64) @ x.astype(np.float64)
    assert np.linalg.norm(d0 - exact) < 0.3 * np.linalg.norm(exact)
    assert not np.array_equal(np.load(tmp_path / "codes0.npy"), np.load(tmp_path / "codes1.npy"))


def test_shard_and_offsets():
    assert shard_tokens(16384, 1, 4) == (4096, 8192)
    with pytest.raises(ValueError):
        shard_tokens(1000, 0, 2)
    assert sr_offset(10, 3, 4) == 43
    # no two (step, rank) pairs share a counter offset
    offs = {sr_offset(s, r, 8) for s in range(50) for r in range(8)}
    assert len(offs) == 50 * 8
    with pytest.raises(ValueError):
        sr_offset((1 << 32) // 2, 1, 2)
    with pytest.raises(ValueError):
        sr_offset(0, 2, 2)
