"""Multi-GPU plumbing for the data-parallel path.

Tokens are independent in both mHC stages, so the forward path shards the token axis:
each rank runs the pre and post stages on its own contiguous block of tokens, and no
collective touches the data path.  The backward's token-local gradients (dX, dF_out) need
no exchange either; its parameter gradients (dphi, db_*, dalpha) are sums over tokens, so
each rank's shard sums are added across ranks with one all-reduce.  The helpers here split
the token axis, sum the parameter gradients, and combine per-rank timings (the job is as
slow as its slowest rank).  They work with any torch.distributed backend (NCCL on GPUs,
gloo in the CPU tests).
"""
from __future__ import annotations


def token_shard(T_total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, stop) block of tokens for `rank`; blocks differ by at most one."""
    if world < 1 or not 0 <= rank < world or T_total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(T_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of `value` over all ranks of the default process group (the value itself when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, steps: int, max_ms: float, world: int) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("time must be positive")
    return world * tokens_per_rank * steps / (max_ms / 1e3)


PARAM_GRADS = ("dphi", "db_pre", "db_post", "db_res", "dalpha")


def allreduce_param_grads(grads: dict, group=None) -> None:
    """Sum mhc_backward's parameter gradients over all ranks, in place.

    grads maps the names in PARAM_GRADS to tensors holding this rank's sums over its own
    token shard.  They travel as one flat bucket in one all-reduce (1.5 MiB of fp32 at
    n = 4, d = 4096), so afterwards every rank holds the gradients over all the job's
    tokens.  A no-op when torch.distributed is not initialised."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return
    ts = [grads[k] for k in PARAM_GRADS]
    flat = torch.cat([t.reshape(-1) for t in ts])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for t in ts:
        n = t.numel()
        t.copy_(flat[off:off + n].view_as(t))
        off += n
