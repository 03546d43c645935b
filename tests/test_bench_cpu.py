"""The benchmark's contract and accounting, checked on the CPU.

The reference arm of ``bench.py`` (the fp64 oracle on the host cores) runs
without a GPU, so its JSON line is checked here end to end; the FLOP
accounting of block masks is checked against its closed forms.
"""
import json
import os
import subprocess
import sys

import torch

from io_aware_exact_25_b200.inputs import WORKLOADS, block_mask, visible_block_fraction

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--ref-rows", "128"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "TFLOPS" and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("long8k_causal")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--warmup", "2"], cwd=ROOT,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0


def test_block_mask_work_fractions():
    H, N = 2, 1000
    nt = (N + 127) // 128
    assert visible_block_fraction(block_mask("ones", H, N), causal=False) == 1.0
    # causal dense: nt(nt-1)/2 full blocks + nt half blocks over nt^2 = 1/2
    assert abs(visible_block_fraction(block_mask("ones", H, N), causal=True) - 0.5) < 1e-12
    assert visible_block_fraction(block_mask("zeros", H, N), causal=True) == 0.0
    # a band of w diagonals on each side plus g global rows/columns
    m = block_mask("local:1,global:1", 1, N)
    dense = torch.zeros(nt, nt)
    for a in range(nt):
        for c in range(nt):
            dense[a, c] = float(abs(a - c) <= 1 or a < 1 or c < 1)
    assert torch.equal(m[0].float(), dense)
    assert abs(visible_block_fraction(m, causal=False) - dense.sum().item() / nt ** 2) < 1e-12


def test_workload_flop_convention():
    w = WORKLOADS["long8k_causal"]
    assert w.fwd_flops() == 4.0 * 2 * 16 * 8192 * 8192 * 128 / 2
    assert w.bwd_flops() == 2.5 * w.fwd_flops()
