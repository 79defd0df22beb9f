"""Host-side logic of running the forward on several GPUs of one node.

The chunked forward is independent per (batch, head) sequence, so N GPUs run N
replicas with no exchange on the data path: in weak scaling every rank processes its
own batch, in strong scaling the sequences of one batch are split across ranks. The
only communication is the timing reduction: whole-job throughput is the units all
ranks processed divided by the slowest rank's device time.
"""
from __future__ import annotations


def shard_sequences(B: int, H: int, world: int, rank: int):
    """Contiguous split of the B*H (batch, head) sequences over `world` ranks.
    Returns the (b, h) pairs of `rank`; the union over ranks is every pair exactly once."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad world / rank")
    n = B * H
    lo = (n * rank) // world
    hi = (n * (rank + 1)) // world
    return [(i // H, i % H) for i in range(lo, hi)]


def aggregate_throughput(local_units: float, local_seconds: float, world: int, device=None):
    """(total units / max seconds over ranks, max seconds) on every rank.
    `local_units` are the units this rank processed in `local_seconds` of device time.
    Uses torch.distributed when world > 1 (any backend: nccl on GPUs, gloo on CPU)."""
    if world == 1:
        return local_units / local_seconds, local_seconds
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_seconds], dtype=torch.float64, device=device)
    u = torch.tensor([local_units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    tmax = float(t.item())
    return float(u.item()) / tmax, tmax
