"""Sequence parallelism across GPUs for long sequences.

"FlashAttention for Efficient Training", section 5.3 (Sequence Parallelism
for Long Contexts): the sequence is cut into chunks held by different GPUs,
and the output for a query needs every key chunk.  The page's formula sums a
softmax per key chunk; read exactly, the output is the logsumexp merge of the
softmax pieces over the chunks -- the same identity as the online softmax and
the split-KV merge (section 6.1).

Layout: every rank holds the queries and dO of the whole sequence (q, do
dense [B, H, N, d]) and one window of the keys (k, v dense [B, H, Nk, d],
key rows [kv_begin, kv_begin + Nk)), the windows of the ranks tiling the
sequence in rank order (``key_windows``).

  forward:  each rank computes the softmax piece of every query over its
            keys (``fa_fwd_partial``: O_r normalised over its keys, lse_r).
            By default the pieces meet in a sum: the lse_r are all-gathered
            (NCCL), every rank rescales its own piece to
            e^(lse_r - lse) O_r (``fa_weight_partial``), one all-reduce adds
            the weighted pieces into O in fp32 and a one-piece
            ``fa_merge_partials`` converts it to bf16.  With
            ``exchange="gather"`` the whole pieces are all-gathered instead
            and every rank merges all of them; per rank that receives
            (W - 1) B H N (d + 1) fp32 values against the sum's
            2 (W - 1) / W B H N d (ring all-reduce) plus the lse gather --
            the same at two ranks, a quarter at eight.
  backward: each rank forms D = dO . O and the scaled lse from the full O
            (``fa_bwd_prepare``), recomputes its key window
            (``fa_bwd_recompute_range``: its dK, dV complete, its part of dQ
            into the fp32 accumulator), the accumulators are summed over the
            ranks (NCCL all-reduce), and ``fa_bwd_finalize`` converts dQ.

The exchanges are the only collectives; the compute steps come from an ops
object (``CudaOps`` on GPUs), so the same orchestration runs under a CPU
test double in multi-process tests.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

TILE = 128


def tile_work(nt: int, causal: bool) -> list:
    """Work of each of the nt key tiles in query-tile x key-tile steps: every
    query tile sees every key tile, or, under the causal mask, key tile t is
    seen by the query tiles t..nt-1 only (the first keys by every query)."""
    return [nt - t for t in range(nt)] if causal else [nt] * nt


def key_windows(N: int, world: int, causal: bool = False) -> list:
    """Key windows [(begin, end)] of the ranks, whole 128-key tiles in rank
    order (a rank may get none).

    Without the mask the ceil(N / 128) tiles are split as evenly as
    possible.  With it the split balances the work (``tile_work``) instead of
    the tile count: boundary r is the tile boundary whose work prefix lies
    closest to r/world of the total, so the early windows, which every query
    sees, are the short ones (two ranks over 64 tiles: 19 and 45 tiles, 1045
    and 1035 steps, where an even tile split gives 1552 and 528)."""
    if world < 1 or N < 0:
        raise ValueError("bad world size or length")
    nt = (N + TILE - 1) // TILE
    if not causal:
        bounds = [r * nt // world for r in range(world + 1)]
    else:
        prefix = [0]
        for wt in tile_work(nt, True):
            prefix.append(prefix[-1] + wt)
        bounds = [0]
        for r in range(1, world):
            target = r * prefix[-1] / world
            t = bounds[-1]
            # inner boundaries stay below the last tile, so the last rank keeps
            # it and an empty window starts on a tile inside the sequence
            while t < nt - 1 and abs(prefix[t + 1] - target) < abs(prefix[t] - target):
                t += 1
            bounds.append(t)
        bounds.append(nt)
    return [(min(a * TILE, N), min(b * TILE, N)) for a, b in zip(bounds, bounds[1:])]


class CudaOps:
    """The per-rank compute steps on the GPU, through the C ABI."""

    def __init__(self):
        from io_aware_exact_25_b200 import binding
        self.b = binding

    def fwd_partial(self, q, k, v, kv_begin, causal, scale, dropout_p, seed):
        return self.b.fwd_partial(q, k, v, kv_begin, causal=causal, scale=scale, dropout_p=dropout_p, seed=seed)

    def merge(self, part_o, part_lse):
        return self.b.merge_partials(part_o, part_lse)

    def weight(self, part_o, all_lse, part):
        return self.b.weight_partial(part_o, all_lse, part)

    def bwd_begin(self, o, do, lse):
        B, H, N, d = o.shape
        ws = torch.empty(self.b.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=o.device)
        self.b.bwd_prepare(o, do, lse, ws)
        return ws

    def bwd_range(self, ws, q, k, v, do, kv_begin, causal, scale, dropout_p, seed):
        return self.b.bwd_recompute_range(q, k, v, do, kv_begin, ws, causal=causal, scale=scale,
                                          dropout_p=dropout_p, seed=seed)

    def dq_accumulator(self, ws, q):
        B, H, N, d = q.shape
        return ws[: self.b.dq_accumulator_bytes(B, H, N, d)].view(torch.float32)

    def bwd_end(self, ws, q, scale):
        return self.b.bwd_finalize(torch.empty_like(q), ws, scale)


def _all_gather(t, world, group):
    flat = torch.empty(world * t.numel(), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(flat, t.contiguous().view(-1), group=group)
    return flat.view((world,) + tuple(t.shape))


def forward(q, k, v, kv_begin, causal=False, scale=None, dropout_p=0.0, seed=0, group=None, ops=None,
            exchange="sum"):
    """Full O and lse on every rank from the ranks' key windows; the ranks'
    windows follow their order in ``group``."""
    if exchange not in ("sum", "gather"):
        raise ValueError("exchange is 'sum' or 'gather'")
    ops = ops or CudaOps()
    d = q.shape[-1]
    scale = scale if scale is not None else d ** -0.5
    part_o, part_lse = ops.fwd_partial(q, k, v, kv_begin, causal, scale, dropout_p, seed)
    world = dist.get_world_size(group)
    if exchange == "gather":
        return ops.merge(_all_gather(part_o, world, group), _all_gather(part_lse, world, group))
    all_lse = _all_gather(part_lse, world, group)
    part_o, lse = ops.weight(part_o, all_lse, dist.get_rank(group))
    dist.all_reduce(part_o, op=dist.ReduceOp.SUM, group=group)
    return ops.merge(part_o.unsqueeze(0), lse.unsqueeze(0))


def backward(q, k, v, o, do, lse, kv_begin, causal=False, scale=None, dropout_p=0.0, seed=0, group=None, ops=None):
    """dQ (full, on every rank) and dK, dV of this rank's key window."""
    ops = ops or CudaOps()
    d = q.shape[-1]
    scale = scale if scale is not None else d ** -0.5
    ws = ops.bwd_begin(o, do, lse)
    dk, dv = ops.bwd_range(ws, q, k, v, do, kv_begin, causal, scale, dropout_p, seed)
    dist.all_reduce(ops.dq_accumulator(ws, q), op=dist.ReduceOp.SUM, group=group)
    dq = ops.bwd_end(ws, q, scale)
    return dq, dk, dv
