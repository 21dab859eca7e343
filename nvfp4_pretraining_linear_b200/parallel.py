"""Data-parallel plumbing for the NVFP4 linear layer (one process per GPU).

Tokens are split across ranks in multiples of 128 rows (so no 16-row RHT / SR
block and no 128-row scale tile straddles two ranks); weights are replicated
and quantised identically on every rank (round-to-nearest is deterministic);
each rank's stochastic rounding uses its own Philox counter offset.  The one
exchange is the weight gradient: an all-reduce (sum) over the data-parallel
group after wgrad, in FP32 (the wgrad GEMM writes FP32 partials, so the sum of
N partials is not rounded to BF16 along the way), started as soon as a linear's
wgrad is enqueued so that it runs during the remaining backward GEMMs.
"""

import torch
import torch.distributed as dist


def shard_tokens(total_tokens, rank, world, multiple=128):
    """[start, stop) of this rank's token rows; every shard a multiple of `multiple`."""
    if total_tokens % (multiple * world):
        raise ValueError("tokens %d do not split into %d shards of %d-row multiples" % (total_tokens, world, multiple))
    per = total_tokens // world
    return rank * per, (rank + 1) * per


def sr_offset(base_offset, rank, world):
    """Philox counter offset of a rank at step `base_offset`: base * world + rank, so no
    two (step, rank) pairs share a counter (offset + 1 per step on every rank keeps them
    apart); it must stay below 2^32."""
    if not 0 <= rank < world:
        raise ValueError("rank %d outside a world of %d" % (rank, world))
    off = int(base_offset) * int(world) + int(rank)
    if off >= 1 << 32:
        raise ValueError("SR offset must stay below 2^32")
    return off


class GradReducer:
    """Sums FP32 weight gradients over the data-parallel group, asynchronously.

    start(g) enqueues an all-reduce of g after the work already on the current
    stream (NCCL runs it on its own stream, so it overlaps what is enqueued next);
    wait() makes the current stream wait for every started all-reduce.  Without an
    initialised process group (one process) both do nothing."""

    def __init__(self, group=None):
        self.group = group
        self.active = dist.is_available() and dist.is_initialized()
        self.pending = []

    def start(self, g):
        if g.dtype != torch.float32:
            raise TypeError("weight gradients are all-reduced in FP32, got %s" % g.dtype)
        if self.active:
            self.pending.append(dist.all_reduce(g, op=dist.ReduceOp.SUM, group=self.group, async_op=True))
        return g

    def wait(self):
        for work in self.pending:
            work.wait()
        self.pending = []


def allreduce_grads(grads, group=None):
    """Sum FP32 weight gradients over the data-parallel group (NCCL on GPU, gloo on CPU)."""
    r = GradReducer(group)
    for g in grads:
        r.start(g)
    r.wait()
    return grads
