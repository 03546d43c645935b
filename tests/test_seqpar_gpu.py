"""The per-rank pieces of sequence parallelism (fa_fwd_partial,
fa_merge_partials, fa_bwd_recompute_range) against the fp64 oracle (GPU).

"FlashAttention for Efficient Training", section 5.3 (Sequence Parallelism
for Long Contexts).  One GPU plays every rank in turn: each key window gets
its own softmax piece and its own backward workspace; the pieces are stacked
and merged, and the windows' fp32 dQ accumulators summed -- the data the
NCCL all-gather and all-reduce of io_aware_exact_25_b200.seqpar exchange
(their bookkeeping is tested over gloo in tests/test_seqpar_gloo.py).
Every element is compared with the bar of tests/parity.py.
"""
import math

import pytest
import torch

import oracle
import parity
from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import make_inputs
from io_aware_exact_25_b200.seqpar import key_windows

pytestmark = pytest.mark.gpu


def _emulate(x, windows, causal, scale, p, seed):
    q, do = x["q"], x["do"]
    parts = [binding.fwd_partial(q, x["k"][:, :, a:b].contiguous(), x["v"][:, :, a:b].contiguous(), a,
                                 causal=causal, scale=scale, dropout_p=p, seed=seed) for a, b in windows]
    o, lse = binding.merge_partials(torch.stack([t[0] for t in parts]), torch.stack([t[1] for t in parts]))
    B, H, N, d = q.shape
    acc_bytes = binding.dq_accumulator_bytes(B, H, N, d)
    total = None
    dks, dvs = [], []
    for a, b in windows:
        ws = torch.empty(binding.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=q.device)
        binding.bwd_prepare(o, do, lse, ws)
        dk, dv = binding.bwd_recompute_range(q, x["k"][:, :, a:b].contiguous(), x["v"][:, :, a:b].contiguous(), do,
                                             a, ws, causal=causal, scale=scale, dropout_p=p, seed=seed)
        dks.append(dk)
        dvs.append(dv)
        acc = ws[:acc_bytes].view(torch.float32)
        if total is None:
            total = ws
        else:
            total[:acc_bytes].view(torch.float32).add_(acc)  # what the all-reduce sums
    dq = binding.bwd_finalize(torch.empty_like(q), total, scale)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    return o, lse, dq, torch.cat(dks, dim=2), torch.cat(dvs, dim=2)


@pytest.mark.parametrize("N,d,causal,world,p", [
    (1000, 128, True, 2, 0.0), (1000, 64, False, 3, 0.0), (777, 128, True, 4, 0.1), (384, 64, True, 8, 0.0),
    (2048, 128, True, 3, 0.0)])
def test_windows_reproduce_the_whole_problem(cuda_device, N, d, causal, world, p):
    """Including ranks whose window no causal query of a tile sees at all,
    windows that end in a ragged tile, and ranks with an empty window."""
    B, H, seed = 1, 2, 23
    x = make_inputs(B, H, N, d, seed=N + world)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = _emulate(xd, key_windows(N, world, causal), causal, scale, p, seed)
    kw = dict(causal=causal, p_drop=p, seed=seed)
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, **kw)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, **kw)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, **kw)
    parity.check("O", o, ro)
    parity.check_lse(lse, rlse)
    if causal and p > 0:
        parity.check("dQ", dq, rdq, exclude_rows=[0])  # reading 11: causal row 0 with dropout
    else:
        parity.check("dQ", dq, rdq)
    parity.check("dK", dk, rdk)
    parity.check("dV", dv, rdv)


def test_one_window_is_the_dense_path(cuda_device):
    """A single window over every key gives the dense kernels' O and lse bit
    for bit (the same softmax pieces, merged once) and their dK, dV."""
    B, H, N, d = 2, 2, 640, 128
    xd = {n: t.to(cuda_device) for n, t in make_inputs(B, H, N, d, seed=5).items()}
    o1, lse1, dq1, dk1, dv1 = _emulate(xd, [(0, N)], True, 1 / math.sqrt(d), 0.0, 0)
    o0, lse0 = binding.fwd(xd["q"], xd["k"], xd["v"], causal=True)
    dq0, dk0, dv0 = binding.bwd(xd["q"], xd["k"], xd["v"], o0, xd["do"], lse0, causal=True)
    torch.cuda.synchronize()
    assert (o1.float() - o0.float()).abs().max().item() <= 2 ** -8
    assert (lse1 - lse0).abs().max().item() <= 1e-5
    assert torch.equal(dk1, dk0) and torch.equal(dv1, dv0)
    assert (dq1.float() - dq0.float()).abs().max().item() <= 2 ** -7
