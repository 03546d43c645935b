"""Split-KV forward (fa_fwd_splitkv) against the fp64 oracle (GPU).

Pieces of the key range are merged by their logsumexp, which is exact in real
arithmetic; the result is held to the same bounds as the plain forward.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _close(name, got, ref):
    """The shared parity bar (tests/parity.py): 2e-2 max abs with the counted
    |ref| >= 4 rounding exception, 5e-3 relative L2."""
    parity.check(name, got, ref)


@pytest.mark.parametrize("N,d,causal,splits", [
    (1024, 128, False, 2), (1024, 128, True, 3), (1000, 64, False, 5), (777, 128, True, 4),
    (2048, 64, True, 16), (256, 128, False, 2), (128, 64, True, 2)])
def test_splitkv_matches_oracle(cuda_device, N, d, causal, splits):
    x = make_inputs(1, 2, N, d, seed=N + splits)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.fwd_splitkv(xd["q"], xd["k"], xd["v"], causal=causal, scale=scale, num_splits=splits)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=causal)
    _close("O", o, ro)
    assert np.abs(lse.cpu().numpy().reshape(rlse.shape) - rlse).max() <= 1e-3


def test_splitkv_with_dropout_and_suggested_splits(cuda_device):
    B, H, N, d = 1, 2, 2048, 128
    x = make_inputs(B, H, N, d, seed=61)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    lib = binding.load()
    splits = lib.fa_splitkv_suggest(B, H, N, d)
    assert splits > 1  # 16 CTAs cannot fill the GPU
    o, lse = binding.fwd_splitkv(xd["q"], xd["k"], xd["v"], causal=True, dropout_p=0.1, seed=4)
    torch.cuda.synchronize()
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], 1 / math.sqrt(d), causal=True, p_drop=0.1, seed=4)
    _close("O", o, ro)
    assert np.abs(lse.cpu().numpy().reshape(rlse.shape) - rlse).max() <= 1e-3
    # the backward accepts the split forward's outputs
    dq, dk, dv = binding.bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, causal=True, dropout_p=0.1, seed=4)
    torch.cuda.synchronize()
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 1 / math.sqrt(d), causal=True, p_drop=0.1,
                                  seed=4)
    _close("dV", dv, rdv)
    _close("dK", dk, rdk)
