"""Multi-GPU plumbing: the one exchange the path has across ranks, and head sharding.

Under data parallelism each rank sees its own batch items, so its max logit
per head covers only those; QK-Clip needs the max over the whole global batch
("Anthology of the SOTA" SOTA-131, "Source": the clip fires for a head whose
max logit exceeds the threshold).  One MAX all-reduce of H floats gives every
rank the global statistic before the clip runs.  Everything else on the path
is independent per batch item / sequence.
"""
from __future__ import annotations


def allreduce_maxlogit(maxlogit, group=None):
    """In place: maxlogit[h] <- max over ranks of maxlogit[h] (NCCL on GPU, gloo on CPU)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(maxlogit, op=dist.ReduceOp.MAX, group=group)
    return maxlogit


def head_range(H: int, world: int, rank: int):
    """Heads [h0, h1) owned by `rank` when H heads are split over `world` ranks.

    Contiguous, as balanced as possible (the first H % world ranks hold one
    more head), covering every head exactly once.
    """
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def qkclip_rescale_heads(geom, W_UQ_shard, W_UKV_shard, maxlogit, tau, h0, clipped=None, gamma=None, stream=None):
    """QK-Clip of one rank's head shard under head (tensor) parallelism.

    The rank holds the contiguous column shards W_UQ[:, h0*d_qk : h1*d_qk] and
    W_UKV[:, h0*(d_c+d_v) : h1*(d_c+d_v)] of heads [h0, h1) and the max logit
    of every head (after the data-parallel MAX all-reduce).  A head's clip
    reads only its own max logit and writes only its own columns, so each
    rank clips its shard with no further exchange.  `clipped` / `gamma`, if
    given, have one entry per local head.
    """
    import dataclasses
    from . import qkclip_rescale
    H_local = W_UQ_shard.shape[-1] // geom.d_qk
    if W_UKV_shard.shape[-1] != H_local * (geom.d_c + geom.d_v):
        raise ValueError("W_UQ and W_UKV shards hold different numbers of heads")
    if not 0 <= h0 <= geom.H - H_local:
        raise ValueError(f"heads [{h0}, {h0 + H_local}) outside the layer's {geom.H}")
    local = dataclasses.replace(geom, H=H_local)
    qkclip_rescale(local, W_UQ_shard, W_UKV_shard, maxlogit[h0:h0 + H_local], tau, clipped, gamma, stream)
