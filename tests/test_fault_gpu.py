"""Failure detection without a GPU fault (GPU).

Every mbarrier wait in the kernels is bounded; when one runs out the kernel
records a timeout in the device error word, every warp leaves its loop, tensor
memory is freed and the kernel returns.  ``fa_debug_fwd_timeout`` runs the real
forward kernel with its producer issuing no K/V load, so the MMA warp's first
wait runs out.  Nothing faults, traps or hangs: the test checks the reported
status and that the context is still usable afterwards.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def test_forced_wait_timeout_is_reported_and_context_survives(cuda_device):
    B, H, N, d = 1, 2, 256, 64
    x = make_inputs(B, H, N, d, seed=90)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    assert binding.device_error() == 0  # the word starts clear
    rc = binding.debug_fwd_timeout(xd["q"], xd["k"], xd["v"], causal=True)
    assert rc == binding.FA_OK
    assert binding.device_error() == 1  # the bounded wait ran out: timeout
    assert binding.device_error() == 0  # reading clears it
    # the same context still runs the real path correctly
    sc = 1.0 / math.sqrt(d)
    o, lse = binding.fwd(xd["q"], xd["k"], xd["v"], causal=True, scale=sc)
    dq, dk, dv = binding.bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, causal=True, scale=sc)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    ro, _ = oracle.forward(x["q"], x["k"], x["v"], sc, causal=True)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], sc, causal=True)
    for got, ref in ((o, ro), (dk, rdk), (dv, rdv)):
        g = got.float().cpu().numpy().reshape(ref.shape)
        assert np.abs(g - ref).max() <= 2e-2
