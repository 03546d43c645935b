"""Multi-GPU helpers: one process per GPU, no collective on the data path.

Every (batch, head) pair of attention is an independent problem ("FlashAttention
for Efficient Training", section 5.3: splitting heads across GPUs), so a job
spreads heads over ranks and needs no exchange of activations.  The only
collective is the max-over-ranks of timings that the benchmark reports.
"""
from __future__ import annotations


def shard_heads(bh: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous range (start, count) of the B*H heads that `rank` owns.

    The first ``bh % world`` ranks own one extra head; every head is owned by
    exactly one rank.
    """
    if world < 1 or not 0 <= rank < world or bh < 0:
        raise ValueError("bad rank/world/head count")
    base, extra = divmod(bh, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None) -> list:
    """Element-wise maximum of a list of floats over all ranks (identity when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def all_ranks_ok(ok: bool, device=None) -> bool:
    """True on every rank iff ``ok`` holds on every rank (identity when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([1.0 if ok else 0.0], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item() > 0.5)


def replica_summary(elapsed_ms: float, e2e_ms: float, stage_ms: list, ok: bool, device=None) -> dict:
    """What one job reports from its replicas: the slowest rank's timings
    (the job is done when the last replica is) and whether every replica's
    output passed its checks.  Every rank takes the same collective steps."""
    times = max_over_ranks([elapsed_ms, e2e_ms] + list(stage_ms), device=device)
    return {"elapsed_ms": times[0], "e2e_ms": times[1], "stage_ms": times[2:],
            "all_ok": all_ranks_ok(ok, device=device)}
