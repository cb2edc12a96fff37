"""Data-parallel plumbing: the one exchange the path has across ranks.

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
