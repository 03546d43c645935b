"""Strided layouts and the autograd wrapper against the fp64 oracle (GPU).

The pages' API takes (batch, seq_len, num_heads, head_dim) tensors
("FlashAttention for Efficient Training", Integration with Frameworks); the
kernels read any [B,H,N,d] view whose head_dim is contiguous.  Same bounds as
the other parity tests.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.attention import flash_attention
from io_aware_exact_25_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _close(name, got, ref):
    """The shared parity bar (tests/parity.py): 2e-2 max abs with the counted
    |ref| >= 4 rounding exception, 5e-3 relative L2."""
    parity.check(name, got, ref)


def _oracle_all(x, scale, causal, p=0.0, seed=0):
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=causal, p_drop=p, seed=seed)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, causal=causal, p_drop=p, seed=seed)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, causal=causal, p_drop=p, seed=seed)
    return ro, rlse, rdq, rdk, rdv


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_bshd_strided_views(cuda_device, d, causal):
    B, H, N = 2, 3, 333
    x = make_inputs(B, H, N, d, seed=51)  # dense [B,H,N,d]; the oracle reads these
    scale = 1.0 / math.sqrt(d)
    # the same values stored (batch, seq, heads, head_dim), viewed as [B,H,N,d]
    bshd = {n: t.transpose(1, 2).contiguous().to(cuda_device) for n, t in x.items()}
    view = {n: t.transpose(1, 2) for n, t in bshd.items()}
    assert not view["q"].is_contiguous()
    o = torch.empty_like(view["q"])
    o, lse = binding.fwd(view["q"], view["k"], view["v"], causal=causal, scale=scale, o=o)
    dq, dk, dv = (torch.empty_like(view["q"]) for _ in range(3))
    binding.bwd(view["q"], view["k"], view["v"], o, view["do"], lse, causal=causal, scale=scale,
                dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    ro, rlse, rdq, rdk, rdv = _oracle_all(x, scale, causal)
    _close("O", o, ro)
    assert np.abs(lse.cpu().numpy().reshape(rlse.shape) - rlse).max() <= 1e-3
    _close("dQ", dq, rdq)
    _close("dK", dk, rdk)
    _close("dV", dv, rdv)


def test_head_slices_of_a_larger_tensor(cuda_device):
    """Views that skip heads (stride over a wider buffer) need no copy."""
    B, H, N, d = 1, 2, 256, 64
    x = make_inputs(B, H, N, d, seed=52)
    big = {n: torch.zeros(B, 2 * H, N, d, dtype=torch.bfloat16, device=cuda_device) for n in x}
    for n, t in x.items():
        big[n][:, ::2] = t.to(cuda_device)
    view = {n: t[:, ::2] for n, t in big.items()}
    o, lse = binding.fwd(view["q"], view["k"], view["v"], causal=True, o=torch.empty_like(x["q"], device=cuda_device))
    torch.cuda.synchronize()
    ro, _ = oracle.forward(x["q"], x["k"], x["v"], 1 / 8, causal=True)
    _close("O", o, ro)


@pytest.mark.parametrize("layout", ["bshd", "bhsd"])
@pytest.mark.parametrize("p", [0.0, 0.1])
def test_flash_attention_autograd(cuda_device, layout, p):
    B, H, N, d = 2, 2, 384, 128
    x = make_inputs(B, H, N, d, seed=53)
    scale = 1.0 / math.sqrt(d)
    to = (lambda t: t.transpose(1, 2).contiguous()) if layout == "bshd" else (lambda t: t.clone())
    q, k, v = (to(x[n]).to(cuda_device).requires_grad_(True) for n in ("q", "k", "v"))
    do = to(x["do"]).to(cuda_device)
    out = flash_attention(q, k, v, causal=True, dropout_p=p, seed=9, layout=layout)
    assert out.shape == q.shape
    out.backward(do)
    torch.cuda.synchronize()
    back = (lambda t: t.transpose(1, 2)) if layout == "bshd" else (lambda t: t)
    ro, _, rdq, rdk, rdv = _oracle_all(x, scale, True, p=p, seed=9)
    _close("O", back(out), ro)
    _close("dQ", back(q.grad), rdq)
    _close("dK", back(k.grad), rdk)
    _close("dV", back(v.grad), rdv)
