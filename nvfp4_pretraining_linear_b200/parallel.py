"""Data-parallel plumbing for the NVFP4 linear layer (one process per GPU).

Tokens are split across ranks in multiples of 128 rows (so no 16-row RHT / SR
block and no 128-row scale tile straddles two ranks); weights are replicated
and quantised identically on every rank (round-to-nearest is deterministic);
each rank's stochastic rounding uses its own Philox counter offset.  The one
exchange is the weight gradient: an all-reduce (sum) over the data-parallel
group after wgrad.
"""

import torch
import torch.distributed as dist


def shard_tokens(total_tokens, rank, world, multiple=128):
    """[start, stop) of this rank's token rows; every shard a multiple of `multiple`."""
    if total_tokens % (multiple * world):
        raise ValueError("tokens %d do not split into %d shards of %d-row multiples" % (total_tokens, world, multiple))
    per = total_tokens // world
    return rank * per, (rank + 1) * per


def sr_offset(base_offset, rank):
    """Philox counter offset of a rank: distinct random words on every rank."""
    off = int(base_offset) + int(rank)
    if off >= 1 << 32:
        raise ValueError("SR offset must stay below 2^32")
    return off


def allreduce_grads(grads, group=None):
    """Sum weight gradients over the data-parallel group (NCCL on GPU, gloo on CPU)."""
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return grads
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
    return grads
