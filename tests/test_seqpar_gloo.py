"""Sequence parallelism across ranks (io_aware_exact_25_b200.seqpar) on CPU
with the gloo backend, world size 2 and 3.

"FlashAttention for Efficient Training", section 5.3 (Sequence Parallelism
for Long Contexts).  The orchestration -- key windows per rank, the
forward exchange (the lse all-gather and the all-reduce of the weighted
pieces, or the all-gather of whole pieces and their merge), the all-reduce
of the dQ accumulators -- runs here unchanged; the per-rank compute steps come from a
CPU double written in fp64 torch from the definition (the CUDA steps are
tested against the oracle on the GPU, tests/test_seqpar_gpu.py).  The
ranks' results must equal the fp64 oracle run on the whole problem.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from io_aware_exact_25_b200.seqpar import key_windows


def test_key_windows_tile_the_sequence():
    for N in (0, 1, 127, 128, 129, 1000, 4096, 8192):
        for world in (1, 2, 3, 8, 40):
            for causal in (False, True):
                w = key_windows(N, world, causal)
                assert len(w) == world and w[0][0] == 0 and w[-1][1] == N
                for (a, b), (c, e) in zip(w, w[1:]):
                    assert b == c and a <= b
                for a, b in w:
                    assert a % 128 == 0 and (b == N or b % 128 == 0)
    with pytest.raises(ValueError):
        key_windows(10, 0)


def _steps(N, a, b, causal):
    """Query-tile x key-tile steps of the window [a, b) by brute force: the
    pairs (query tile i, key tile t) of which some query sees some key."""
    nt = (N + 127) // 128
    return sum(1 for t in range(a // 128, (b + 127) // 128) for i in range(nt) if not causal or i >= t)


def test_causal_windows_balance_the_work():
    """Under the causal mask no contiguous tile split has a smaller largest
    window (brute force over every split for small cases), and the long8k
    split at 2, 4 and 8 ranks stays within a few percent of even."""
    import itertools
    for nt in (1, 2, 5, 9, 16):
        N = nt * 128
        for world in (2, 3, 4):
            got = max(_steps(N, a, b, True) for a, b in key_windows(N, world, True))
            best = min(max(_steps(N, 128 * x, 128 * y, True) for x, y in zip((0,) + c, c + (nt,)))
                       for c in itertools.combinations_with_replacement(range(nt + 1), world - 1))
            # closest-prefix boundaries are within one tile's work of the best split
            assert got <= best + nt, (nt, world, got, best)
    total = _steps(8192, 0, 8192, True)
    for world, slack in ((2, 1.01), (4, 1.04), (8, 1.12)):
        per = [_steps(8192, a, b, True) for a, b in key_windows(8192, world, True)]
        assert sum(per) == total and max(per) <= slack * total / world, (world, per)
    # the even tile split it replaces: 1552 and 528 steps at two ranks
    assert [_steps(8192, a, b, True) for a, b in key_windows(8192, 2)] == [1552, 528]


class CpuOps:
    """fp64 torch double of the per-rank compute steps (same contract as
    seqpar.CudaOps), written from the definition with global row statistics."""

    def __init__(self, keep):
        self.keep = keep  # dropout keep mask [B, H, N, N] as 0/1 (all ones without dropout)

    def _scores(self, q, k, kv_begin, causal, scale):
        N, nk = q.shape[2], k.shape[2]
        s = (q @ k.transpose(-1, -2)) * scale
        if causal:
            i = torch.arange(N).view(N, 1)
            j = kv_begin + torch.arange(nk).view(1, nk)
            s = s.masked_fill(j > i, float("-inf"))
        return s

    def fwd_partial(self, q, k, v, kv_begin, causal, scale, p, seed):
        q, k, v = q.double(), k.double(), v.double()
        nk = k.shape[2]
        s = self._scores(q, k, kv_begin, causal, scale)
        lse = torch.logsumexp(s, dim=-1)
        prob = torch.where(torch.isneginf(lse)[..., None], torch.zeros_like(s), torch.exp(s - lse[..., None]))
        z = self.keep[..., kv_begin:kv_begin + nk] / (1.0 - p)
        return (prob * z) @ v, lse

    def merge(self, all_o, all_lse):
        lse = torch.logsumexp(all_lse, dim=0)
        w = torch.where(torch.isneginf(all_lse), torch.zeros_like(all_lse), torch.exp(all_lse - lse))
        return (w[..., None] * all_o).sum(0), lse

    def weight(self, part_o, all_lse, part):
        lse = torch.logsumexp(all_lse, dim=0)
        mine = all_lse[part]
        w = torch.where(torch.isneginf(mine), torch.zeros_like(mine), torch.exp(mine - lse))
        return part_o * w[..., None], lse

    def bwd_begin(self, o, do, lse):
        return {"D": (do.double() * o.double()).sum(-1), "lse": lse.double(),
                "acc": torch.zeros(o.shape, dtype=torch.float64)}

    def bwd_range(self, ws, q, k, v, do, kv_begin, causal, scale, p, seed):
        q, k, v, do = q.double(), k.double(), v.double(), do.double()
        nk = k.shape[2]
        s = self._scores(q, k, kv_begin, causal, scale)
        prob = torch.exp(s - ws["lse"][..., None])
        z = self.keep[..., kv_begin:kv_begin + nk] / (1.0 - p)
        dp = (do @ v.transpose(-1, -2)) * z
        ds = prob * (dp - ws["D"][..., None])
        ws["acc"] += scale * (ds @ k)
        return scale * (ds.transpose(-1, -2) @ q), (prob * z).transpose(-1, -2) @ do

    def dq_accumulator(self, ws, q):
        return ws["acc"]

    def bwd_end(self, ws, q, scale):
        return ws["acc"]


# name: (causal, dropout p, forward exchange)
CASES = {"causal": (True, 0.0, "sum"), "noncausal_dropout": (False, 0.2, "sum"),
         "causal_gather": (True, 0.0, "gather")}


def _worker(rank, world, out_dir, case):
    from datetime import timedelta
    # a file store: no TCP port to collide with other tests
    dist.init_process_group("gloo", init_method="file://" + os.path.join(out_dir, "store"), rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    try:
        import oracle
        from io_aware_exact_25_b200 import seqpar
        from io_aware_exact_25_b200.inputs import make_inputs
        causal, p, exchange = CASES[case]
        B, H, N, d, seed = 1, 2, 300, 16, 7
        x = make_inputs(B, H, N, d, seed=61)
        keep = torch.from_numpy(oracle.dropout_mask(B, H, N, p, seed).astype(np.float64)).view(B, H, N, N)
        ops = CpuOps(keep)
        kb, ke = seqpar.key_windows(N, world, causal)[rank]
        k, v = x["k"][:, :, kb:ke], x["v"][:, :, kb:ke]
        scale = 0.3
        o, lse = seqpar.forward(x["q"], k, v, kb, causal=causal, scale=scale, dropout_p=p, seed=seed, ops=ops,
                                exchange=exchange)
        dq, dk, dv = seqpar.backward(x["q"], k, v, o, x["do"], lse, kb, causal=causal, scale=scale, dropout_p=p,
                                     seed=seed, ops=ops)
        for name, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
            np.save(os.path.join(out_dir, f"{name}{rank}.npy"), t.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", sorted(CASES))
def test_ranks_reproduce_the_whole_problem(tmp_path, world, case):
    mp.start_processes(_worker, args=(world, str(tmp_path), case), nprocs=world,
                       start_method="spawn", join=True)
    import oracle
    from io_aware_exact_25_b200.inputs import make_inputs
    causal, p, _ = CASES[case]
    B, H, N, d, seed = 1, 2, 300, 16, 7
    x = make_inputs(B, H, N, d, seed=61)
    kw = dict(causal=causal, p_drop=p, seed=seed)
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], 0.3, **kw)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], 0.3, **kw)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 0.3, **kw)
    ld = lambda n, r: np.load(tmp_path / f"{n}{r}.npy")
    for r in range(world):  # every rank holds the full O, lse and dQ
        assert np.max(np.abs(ld("o", r).reshape(ro.shape) - ro)) < 1e-12
        assert np.max(np.abs(ld("lse", r).reshape(rlse.shape) - rlse)) < 1e-12
        assert np.max(np.abs(ld("dq", r).reshape(rdq.shape) - rdq)) < 1e-11
    dk = np.concatenate([ld("dk", r) for r in range(world)], axis=2).reshape(rdk.shape)
    dv = np.concatenate([ld("dv", r) for r in range(world)], axis=2).reshape(rdv.shape)
    assert np.max(np.abs(dk - rdk)) < 1e-11 and np.max(np.abs(dv - rdv)) < 1e-11
    assert math.isfinite(float(dk.sum()))
