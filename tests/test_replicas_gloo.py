"""Multi-process (world_size 2, gloo, CPU) checks of the replica path.

Heads are independent, so ranks that each compute a disjoint shard of heads
reproduce the full result with no exchange; the only collective is the
max-over-ranks of timings.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from io_aware_exact_25_b200.replicas import max_over_ranks, replica_summary, shard_heads


def test_shard_heads_covers_every_head_once():
    for bh in (0, 1, 5, 32, 33):
        for world in (1, 2, 3, 8):
            owned = []
            for r in range(world):
                s, c = shard_heads(bh, r, world)
                owned += list(range(s, s + c))
            assert owned == list(range(bh))
    with pytest.raises(ValueError):
        shard_heads(4, 2, 2)


def _worker(rank, world, out_dir):
    dist.init_process_group("gloo", init_method="file://" + os.path.join(out_dir, "store"), rank=rank,
                            world_size=world)
    try:
        import oracle
        from io_aware_exact_25_b200.inputs import make_inputs
        x = make_inputs(1, 5, 64, 8, seed=3)
        start, count = shard_heads(5, rank, world)
        o, lse = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=True,
                                heads=list(range(start, start + count)))
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o)
        # timing reduction: every rank sees the slowest rank's numbers
        m = max_over_ranks([1.0 + rank, 10.0 - rank])
        np.save(os.path.join(out_dir, f"m{rank}.npy"), np.array(m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_head_shards_reproduce_full_result(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    import oracle
    from io_aware_exact_25_b200.inputs import make_inputs
    x = make_inputs(1, 5, 64, 8, seed=3)
    full, _ = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=True)
    parts = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)])
    assert np.array_equal(parts, full)
    for r in range(world):
        assert np.load(tmp_path / f"m{r}.npy").tolist() == [2.0, 10.0]


def test_max_over_ranks_without_process_group():
    assert max_over_ranks([1.5, 2.0]) == [1.5, 2.0]


def _summary_worker(rank, world, out_dir):
    dist.init_process_group("gloo", init_method="file://" + os.path.join(out_dir, "store"), rank=rank,
                            world_size=world)
    try:
        # what bench.py's torchrun path reports: rank 1 is slower in the timed
        # region, rank 0 in the end-to-end leg, and rank 1's outputs failed
        s = replica_summary(10.0 + rank, 50.0 - rank, [1.0 + rank, 2.0 - rank], ok=(rank == 0))
        np.save(os.path.join(out_dir, f"s{rank}.npy"),
                np.array([s["elapsed_ms"], s["e2e_ms"]] + s["stage_ms"] + [float(s["all_ok"])]))
        s2 = replica_summary(1.0, 1.0, [], ok=True)
        np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([float(s2["all_ok"])]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_bench_replica_summary_over_two_ranks(tmp_path):
    """The bench's rank bookkeeping: every rank ends with the slowest rank's
    times, and one failing replica fails the job on every rank."""
    world = 2
    mp.start_processes(_summary_worker, args=(world, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        assert np.load(tmp_path / f"s{r}.npy").tolist() == [11.0, 50.0, 2.0, 2.0, 0.0]
        assert np.load(tmp_path / f"t{r}.npy").tolist() == [1.0]
