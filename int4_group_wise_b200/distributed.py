"""The Hessian with its calibration rows split across GPUs (one process per GPU).

The exchange step of the path: H = X^T X / n is a sum over the n calibration
rows ("Opt.Gear-QAT" blog, section 2: layer sensitivity from calibration
activations), so each rank computes the partial of its own contiguous shard of
rows, already divided by the global n (qat4_hessian_partial), and one sum
all-reduce over NCCL (NVLink / NVSwitch) gives every rank the whole H.  The
scale search and the LSQ step that follow shard by rows of W with no
collective.

Only plumbing lives here: the shard bounds and the all-reduce.  The arithmetic
is the library's kernel; torch.distributed moves the partials.
"""
from __future__ import annotations


def shard_rows(n: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [lo, hi) of rank `rank` among `world` near-equal contiguous shards of n rows."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard request")
    return n * rank // world, n * (rank + 1) // world


def allreduce_partials(H_partial, group=None):
    """Sum the ranks' partial Hessians in place (every rank ends with the full H)."""
    import torch.distributed as dist
    dist.all_reduce(H_partial, op=dist.ReduceOp.SUM, group=group)
    return H_partial


def hessian_sharded(X_shard, n_total: int, group=None, H=None, workspace=None, stream=None):
    """H of all n_total calibration rows from this rank's shard X_shard (bf16 [n_r, C], on this
    rank's GPU): the shard's partial on the tensor cores, then one NCCL all-reduce."""
    import torch

    from . import hessian_partial
    if X_shard.shape[0] < 1:
        raise ValueError("every rank needs at least one calibration row")
    H = hessian_partial(X_shard, n_total, H=H, workspace=workspace, stream=stream)
    s = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.stream(s):
        allreduce_partials(H, group)
    return H
