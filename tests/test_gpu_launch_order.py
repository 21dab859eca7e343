"""Launch order: the quantise pass is a programmatic dependent of its amax pass, and
every pair GEMM of the kernel before it (both overlap their set-up with that kernel's
last CTAs and wait for it before they touch its results).  Chains of dependent calls
enqueued back to back must give the same bytes as the same calls with a device
synchronisation between each, including when the input of a quantisation was written
by the launch right before it (a GEMM output, or a torch copy)."""

import pytest
import torch

from nvfp4_pretraining_linear_b200 import api, synthetic

pytestmark = pytest.mark.gpu

SIGNS = 0x5A3C


def chain(x, w, sync):
    """fprop, then the output quantised as the next layer's activation (RHT col) and as
    a gradient (SR), a GEMM on each of those, and a wgrad-shaped GEMM."""
    def s():
        if sync:
            torch.cuda.synchronize()
    wq_row, wq_col = api.quantize_weight(w)
    s()
    xq_row, xq_col = api.quantize(x, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS)
    s()
    y = api.gemm(xq_row, wq_row)                               # written by a GEMM ...
    s()
    yq_row, yq_col = api.quantize(y, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS)   # ... read here
    s()
    gq_row, gq_col = api.quantize(y, emit_row=True, emit_col=True, stochastic=True, rht_col=True, seed=7,
                                  offset=1, rht_signs=SIGNS)
    s()
    z = api.gemm(yq_row, yq_row, out_dtype=torch.float32)
    s()
    dx = api.gemm(gq_row, wq_col)
    s()
    dw = api.gemm(gq_col, xq_col, out_dtype=torch.float32)
    s()
    return [xq_row, xq_col, yq_row, yq_col, gq_row, gq_col], [y, z, dx, dw]


def same_bytes(qa, qb):
    return all(torch.equal(a.codes, b.codes) and torch.equal(a.scales, b.scales)
               and torch.equal(a.tensor_scale, b.tensor_scale) for a, b in zip(qa, qb))


@pytest.mark.parametrize("M,K,N", [(1024, 768, 1280), (2304, 1024, 3328)])
def test_back_to_back_chain_matches_serialised(M, K, N):
    x = synthetic.normal((M, K), 1.0, seed=61, device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    w = synthetic.normal((N, K), 0.02, seed=62, device="cuda")
    q_ref, o_ref = chain(x, w, sync=True)
    for _ in range(3):
        q, o = chain(x, w, sync=False)
        torch.cuda.synchronize()
        assert same_bytes(q, q_ref)
        assert all(torch.equal(a, b) for a, b in zip(o, o_ref))
    api.get_status()


def test_quantise_reads_input_written_just_before():
    """A torch copy writes x right before each quantisation (no synchronisation): the
    quantise pass, which starts loading x while its amax pass finishes, must see the new
    values every time."""
    M, K = 2048, 2048
    srcs = [synthetic.student_t((M, K), 3, 0.1, seed=70 + i, device="cuda") for i in range(4)]
    refs = [api.quantize(s, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS) for s in srcs]
    torch.cuda.synchronize()
    x = torch.empty_like(srcs[0])
    outs = []
    for i in range(12):
        x.copy_(srcs[i % 4])
        outs.append(api.quantize(x, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS))
    torch.cuda.synchronize()
    for i, q in enumerate(outs):
        assert same_bytes(q, refs[i % 4]), i
    api.get_status()


def test_step_captured_in_cuda_graph_matches_eager():
    """The linear step's calls captured into a CUDA graph (the memsets become graph
    nodes, the programmatic-dependent launches programmatic edges) and replayed give
    the bytes of the eager calls, and a replay after the input is rewritten in place
    follows the new values."""
    M, K, N = 1024, 768, 1280
    x = synthetic.normal((M, K), 1.0, seed=81, device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    x2 = synthetic.normal((M, K), 1.0, seed=82, device="cuda", outlier_frac=0.001, outlier_mult=100.0)
    w = synthetic.normal((N, K), 0.02, seed=83, device="cuda")
    dy = synthetic.normal((M, N), 1e-3, seed=84, device="cuda")
    E = api.QTensor.empty
    q = [E(N, K), E(K, N), E(M, K), E(K, M), E(M, N), E(N, M)]     # Wq, Xq, dYq: row, col
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")

    def step():
        api.quantize(w, emit_row=True, emit_col=True, block_2d=True, out_row=q[0], out_col=q[1])
        api.quantize(x, emit_row=True, emit_col=True, rht_col=True, rht_signs=SIGNS, out_row=q[2], out_col=q[3])
        api.gemm(q[2], q[0], out=y)
        api.quantize(dy, emit_row=True, emit_col=True, stochastic=True, rht_col=True, seed=5, offset=2,
                     rht_signs=SIGNS, out_row=q[4], out_col=q[5])
        api.gemm(q[4], q[1], out=dx)
        api.gemm(q[5], q[3], out=dw)

    def snapshot():
        torch.cuda.synchronize()
        return ([(t.codes.clone(), t.scales.clone(), t.tensor_scale.clone()) for t in q],
                [y.clone(), dx.clone(), dw.clone()])

    def same(a, b):
        return all(all(torch.equal(u, v) for u, v in zip(ta, tb)) for ta, tb in zip(a[0], b[0])) and \
            all(torch.equal(u, v) for u, v in zip(a[1], b[1]))

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()                                   # eager; also creates stream s's workspace
    ref = snapshot()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for t in q:
        t.codes.fill_(0x5A)
        t.scales.fill_(0x33)
    y.fill_(7.0)
    g.replay()
    assert same(snapshot(), ref)
    x.copy_(x2)
    g.replay()
    replayed = snapshot()
    with torch.cuda.stream(s):
        step()
    assert same(replayed, snapshot())
    assert not torch.equal(replayed[1][0], ref[1][0])      # the new input did reach the output
    api.get_status()
