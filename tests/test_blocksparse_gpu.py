"""Block-sparse attention (fa_fwd_blocksparse / fa_bwd_blocksparse) against the
fp64 oracle with the same block mask (GPU).

"FlashAttention for Efficient Training" section 3.2 (Block-Sparse Attention
Support): zero blocks of a mask over 128 x 128 tiles are skipped.  Rows that
see no key get O = 0 and lse = -inf; keys no query sees get dK = dV = 0.
Bounds as for the dense path (tests/parity.py): max |err| <= 2e-2 with the
counted |ref| >= 4 rounding exception, relative L2 <= 5e-3, lse within 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import block_mask, make_inputs, sample_rows

pytestmark = pytest.mark.gpu


_check = parity.check
_check_lse = parity.check_lse


def _run(x, mask, causal, scale, p=0.0, seed=0, dev="cuda"):
    xd = {n: t.to(dev) for n, t in x.items()}
    md = mask.to(dev)
    o, lse = binding.fwd(xd["q"], xd["k"], xd["v"], causal=causal, scale=scale, dropout_p=p, seed=seed,
                         block_mask=md)
    dq, dk, dv = binding.bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, causal=causal, scale=scale,
                             dropout_p=p, seed=seed, block_mask=md)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    return o, lse, dq, dk, dv


def _compare_all(x, mask, causal, scale, out, p=0.0, seed=0):
    o, lse, dq, dk, dv = out
    bm = mask.numpy()
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=causal, p_drop=p, seed=seed, block_mask=bm)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, causal=causal, p_drop=p, seed=seed,
                                  block_mask=bm)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, causal=causal, p_drop=p, seed=seed,
                                  block_mask=bm)
    _check("O", o, ro)
    _check_lse(lse, rlse)
    _check("dQ", dq, rdq)
    _check("dK", dk, rdk)
    _check("dV", dv, rdv)


@pytest.mark.parametrize("N,d,causal,kind,shared", [
    (1024, 64, False, "random:0.4", False),
    (1000, 128, True, "random:0.5", False),     # ragged last tile
    (777, 64, True, "local:1,global:1", True),
    (1280, 128, False, "local:2,global:0", True),
    (640, 128, False, "random:0.25", True),     # sparse enough to empty whole rows and columns
    (300, 64, True, "ones", True),
])
def test_blocksparse_matches_oracle(cuda_device, N, d, causal, kind, shared):
    B, H = 2, 3
    x = make_inputs(B, H, N, d, seed=N + d)
    mask = block_mask(kind, 1 if shared else H, N, seed=N)
    scale = 1.0 / math.sqrt(d)
    out = _run(x, mask, causal, scale, dev=cuda_device)
    _compare_all(x, mask, causal, scale, out)


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_with_dropout(cuda_device, d):
    B, H, N = 1, 2, 896
    x = make_inputs(B, H, N, d, seed=70 + d)
    mask = block_mask("random:0.5", H, N, seed=71)
    scale = 1.0 / math.sqrt(d)
    out = _run(x, mask, True, scale, p=0.15, seed=9, dev=cuda_device)
    _compare_all(x, mask, True, scale, out, p=0.15, seed=9)


def test_empty_query_and_key_tiles(cuda_device):
    """A query tile with no visible block: O = 0, lse = -inf, dQ = 0; a key tile
    no query tile sees: dK = dV = 0."""
    B, H, N, d = 1, 2, 512, 128
    x = make_inputs(B, H, N, d, seed=80)
    mask = torch.ones((H, 4, 4), dtype=torch.uint8)
    mask[0, 1, :] = 0          # head 0: query tile 1 sees nothing
    mask[1, :, 2] = 0          # head 1: nobody sees key tile 2
    mask[1, 3, :] = 0          # head 1: the last query tile sees nothing
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = out = _run(x, mask, False, scale, dev=cuda_device)
    assert torch.all(o[0, 0, 128:256] == 0) and torch.all(torch.isneginf(lse[0, 0, 128:256]))
    assert torch.all(dq[0, 0, 128:256] == 0)
    assert torch.all(dk[0, 1, 256:384] == 0) and torch.all(dv[0, 1, 256:384] == 0)
    assert torch.all(o[0, 1, 384:] == 0) and torch.all(dq[0, 1, 384:] == 0)
    _compare_all(x, mask, False, scale, out)


def test_all_zero_mask(cuda_device):
    B, H, N, d = 1, 2, 300, 64
    x = make_inputs(B, H, N, d, seed=81)
    mask = block_mask("zeros", 1, N)
    o, lse, dq, dk, dv = _run(x, mask, True, 0.125, dev=cuda_device)
    assert torch.all(torch.isneginf(lse))
    for t in (o, dq, dk, dv):
        assert torch.all(t == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_equals_dense_kernels(cuda_device, causal):
    """An all-ones mask runs the same tiles in the same order as the dense
    kernels: O, lse, dK and dV agree bit for bit (dQ is summed across CTAs in
    an order that may differ, so it is held to the parity bound)."""
    B, H, N, d = 2, 2, 1000, 128
    x = make_inputs(B, H, N, d, seed=82)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    mask = block_mask("ones", 1, N).to(cuda_device)
    sc = 1.0 / math.sqrt(d)
    o1, l1 = binding.fwd(xd["q"], xd["k"], xd["v"], causal=causal, scale=sc)
    o2, l2 = binding.fwd(xd["q"], xd["k"], xd["v"], causal=causal, scale=sc, block_mask=mask)
    g1 = binding.bwd(xd["q"], xd["k"], xd["v"], o1, xd["do"], l1, causal=causal, scale=sc)
    g2 = binding.bwd(xd["q"], xd["k"], xd["v"], o2, xd["do"], l2, causal=causal, scale=sc, block_mask=mask)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert (g1[0].float() - g2[0].float()).abs().max().item() <= 2e-2


def test_blocksparse_long_sequence_sampled(cuda_device):
    """N = 16384 with a sliding-window + global pattern (10% of blocks):
    sampled query rows (O, lse, dQ) and key rows (dK, dV) against the oracle."""
    B, H, N, d = 1, 4, 16384, 128
    x = make_inputs(B, H, N, d, seed=83, qkv_scale=0.5)
    mask = block_mask("local:4,global:2", 1, N)
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = _run(x, mask, True, scale, dev=cuda_device)
    rows = sample_rows(N, 48, seed=83)
    heads = [0, 3]
    bm = mask.numpy()
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=True, heads=heads, rows=rows, block_mask=bm)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, causal=True, heads=heads, rows=rows,
                                  block_mask=bm)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, causal=True, heads=heads, keys=rows,
                                  block_mask=bm)
    _check("O", o[0][heads][:, rows], ro)
    _check_lse(lse[0][heads][:, rows], rlse)
    _check("dQ", dq[0][heads][:, rows], rdq)
    _check("dK", dk[0][heads][:, rows], rdk)
    _check("dV", dv[0][heads][:, rows], rdv)


def test_autograd_wrapper_with_block_mask(cuda_device):
    from io_aware_exact_25_b200.attention import flash_attention
    B, H, N, d = 1, 2, 512, 64
    x = make_inputs(B, H, N, d, seed=84)
    mask = block_mask("random:0.5", H, N, seed=85)
    q, k, v = (x[n].to(cuda_device).transpose(1, 2).contiguous().requires_grad_(True) for n in ("q", "k", "v"))
    o = flash_attention(q, k, v, causal=True, block_mask=mask.to(cuda_device).bool())
    o.backward(x["do"].to(cuda_device).transpose(1, 2))
    torch.cuda.synchronize()
    bm = mask.numpy()
    sc = 1.0 / math.sqrt(d)
    ro, _ = oracle.forward(x["q"], x["k"], x["v"], sc, causal=True, block_mask=bm)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], sc, causal=True, block_mask=bm)
    _check("O", o.transpose(1, 2), ro)
    _check("dQ", q.grad.transpose(1, 2), rdq)


def test_staged_blocksparse_backward_equals_one_call(cuda_device):
    """fa_bwd_prepare + fa_bwd_recompute_blocksparse + fa_bwd_finalize is
    fa_bwd_blocksparse."""
    B, H, N, d = 1, 2, 700, 128
    x = make_inputs(B, H, N, d, seed=86)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    mask = block_mask("random:0.6", H, N, seed=87).to(cuda_device)
    sc = 1.0 / math.sqrt(d)
    o, lse = binding.fwd(xd["q"], xd["k"], xd["v"], causal=True, scale=sc, block_mask=mask)
    dq1, dk1, dv1 = binding.bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, causal=True, scale=sc,
                                block_mask=mask)
    lib = binding.load()
    wsb = binding.bwd_workspace_size(B, H, N, d)
    work = torch.empty(wsb, dtype=torch.uint8, device=cuda_device)
    dq2, dk2, dv2 = (torch.empty_like(xd["q"]) for _ in range(3))
    s = torch.cuda.current_stream().cuda_stream
    P = binding._ptr
    assert lib.fa_bwd_prepare(P(o), P(xd["do"]), P(lse), B, H, N, d, P(work), wsb, s) == 0
    assert lib.fa_bwd_recompute_blocksparse(P(xd["q"]), P(xd["k"]), P(xd["v"]), P(xd["do"]), P(dk2), P(dv2), B, H, N,
                                            d, sc, 1, 0.0, 0, P(mask), H, P(work), wsb, s) == 0
    assert lib.fa_bwd_finalize(P(dq2), B, H, N, d, sc, P(work), wsb, s) == 0
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert (dq1.float() - dq2.float()).abs().max().item() <= 2e-2
