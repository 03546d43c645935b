"""``flash_attention(Q, K, V)``: the pages' framework-level API on the C ABI.

"FlashAttention for Efficient Training", Integration with Frameworks, shows
attention called as ``output = flash_attention(Q, K, V)`` on tensors laid out
(batch, seq_len, num_heads, head_dim), with autograd supplying the backward
through the library's own backward kernels.  This module is that call: a
``torch.autograd.Function`` whose forward is ``fa_fwd_strided`` and whose
backward is ``fa_bwd_strided`` (their block-sparse forms with a block mask),
on strided views of the caller's tensors, so
no layout copies are made.  torch supplies memory, streams and autograd
bookkeeping; every step of the computation runs in the CUDA library.
"""
from __future__ import annotations

import math

import torch

from . import binding


def _usable(t) -> bool:
    """A view the kernels can address directly: unit last stride and 16-byte
    aligned row starts."""
    return t.stride(-1) == 1 and all((s * t.element_size()) % 16 == 0 for s in t.stride()[:3]) \
        and t.data_ptr() % 16 == 0


class _FlashAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, dropout_p, seed, block_mask):
        o = torch.empty_like(q)  # same (possibly strided) layout as q
        o, lse = binding.fwd(q, k, v, causal=causal, scale=scale, dropout_p=dropout_p, seed=seed, o=o,
                             block_mask=block_mask)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.args = (causal, scale, dropout_p, seed, block_mask)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        causal, scale, dropout_p, seed, block_mask = ctx.args
        if not _usable(do):
            do = do.contiguous()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        binding.bwd(q, k, v, o, do, lse, causal=causal, scale=scale, dropout_p=dropout_p, seed=seed,
                    dq=dq, dk=dk, dv=dv, block_mask=block_mask)
        return dq, dk, dv, None, None, None, None, None


def flash_attention(q, k, v, causal: bool = False, dropout_p: float = 0.0, scale: float | None = None,
                    seed: int | None = None, layout: str = "bshd", block_mask=None):
    """Exact attention softmax(scale * Q K^T [+ causal]) V with autograd.

    q, k, v: bf16 CUDA tensors, (batch, seq_len, num_heads, head_dim) for
    ``layout="bshd"`` (the pages' layout) or (batch, num_heads, seq_len,
    head_dim) for ``layout="bhsd"``; head_dim 64 or 128; any strides with a
    contiguous head_dim and 16-byte aligned rows (others are copied once).
    Returns the output in the same layout.  ``seed`` fixes the dropout mask
    (drawn from torch's generator when None); the backward regenerates the
    same mask.  ``block_mask`` (uint8 or bool CUDA tensor [1 or H, nt, nt],
    nt = ceil(seq_len / 128)) makes the attention block-sparse
    ("FlashAttention for Efficient Training" section 3.2): zero blocks are
    skipped, rows that see no key get a zero output.
    """
    if layout not in ("bshd", "bhsd"):
        raise ValueError("layout is 'bshd' or 'bhsd'")
    if layout == "bshd":
        q, k, v = (t.transpose(1, 2) for t in (q, k, v))
    q, k, v = (t if _usable(t) else t.contiguous() for t in (q, k, v))
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if seed is None:
        seed = int(torch.randint(0, 2 ** 62, (1,)).item()) if dropout_p > 0 else 0
    if block_mask is not None and not block_mask.is_contiguous():
        block_mask = block_mask.contiguous()
    o = _FlashAttention.apply(q, k, v, bool(causal), float(scale), float(dropout_p), int(seed), block_mask)
    return o.transpose(1, 2) if layout == "bshd" else o
