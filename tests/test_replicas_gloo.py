"""Multi-process (world_size 2, gloo, CPU) checks of the replica path.

Heads are independent, so ranks that each compute a disjoint shard of heads
reproduce the full result with no exchange; the only collective is the
max-over-ranks of timings.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from io_aware_exact_25_b200.replicas import max_over_ranks, shard_heads


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


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
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
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
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
