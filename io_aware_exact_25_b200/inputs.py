"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and rounds them to bf16; it holds none of
the attention arithmetic.  Both the CUDA path and the fp64 oracle consume the
same bf16 tensors it returns.

Recipe (the same for every workload):
  * ``g = torch.Generator().manual_seed(seed)`` on the CPU;
  * draw fp32 ``randn`` tensors of shape ``[B, H, N, d]`` in the order
    Q, K, V, dO;
  * ``qkv_scale`` multiplies Q, K and V (exact for 0.5);
  * ``offset_norm > 0``: draw ``g_h ~ N(0, I_d)`` per head (after dO), set
    ``u_h = offset_norm * g_h / |g_h|`` and add the same ``u_h`` to every row
    of both Q and K of head h (peaked softmax rows);
  * round each tensor to bf16 (round-to-nearest-even).

The named workloads stand in for the pages' model-level benchmarks (BERT,
GPT-3, ViT at sequence lengths 512-2048, and the 32K/64K long-context
examples), none of which can be reproduced without models or data.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    p_drop: float
    seed: int
    qkv_scale: float = 1.0
    offset_norm: float = 0.0
    # variable-length batch: the B sequence lengths (N is the longest); empty
    # for a dense [B, H, N, d] workload
    lens: tuple = ()

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved when causal (the attention FLOP convention);
        a variable-length batch sums 4*H*L^2*d over its sequences."""
        if self.lens:
            f = sum(4.0 * self.H * L * L * self.d for L in self.lens)
        else:
            f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f

    def bwd_flops(self) -> float:
        """2.5x the forward (five GEMMs against two)."""
        return 2.5 * self.fwd_flops()


def varlen_lengths(count: int, lo: int, hi: int, seed: int) -> tuple:
    """``count`` sequence lengths drawn uniformly from [lo, hi] by a torch
    generator seeded with ``2000 + seed`` (a mixed-length training batch)."""
    g = torch.Generator().manual_seed(2000 + int(seed))
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (count,), generator=g))


_MIX = varlen_lengths(16, 512, 8192, 6)

WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 128, 64, False, 0.0, 0),
    "train2k": Workload("train2k", 4, 16, 2048, 64, False, 0.0, 1),
    "train2k_causal": Workload("train2k_causal", 4, 16, 2048, 64, True, 0.0, 1),
    "long8k_causal": Workload("long8k_causal", 2, 16, 8192, 128, True, 0.0, 2, qkv_scale=0.5),
    "long32k_causal": Workload("long32k_causal", 1, 16, 32768, 128, True, 0.0, 3, offset_norm=2.0),
    "long64k_causal_dropout": Workload("long64k_causal_dropout", 1, 8, 65536, 128, True, 0.1, 4),
    # few query tiles (64 CTAs of work for 148 SMs): the split-KV case
    "smallbatch16k": Workload("smallbatch16k", 1, 1, 16384, 128, False, 0.0, 5),
    # a variable-length batch: 16 sequences of 512-8192 tokens packed back to
    # back (token-major), causal, d = 128
    "varlen_mix": Workload("varlen_mix", len(_MIX), 16, max(_MIX), 128, True, 0.0, 6, lens=_MIX),
}


def make_inputs(B: int, H: int, N: int, d: int, seed: int, qkv_scale: float = 1.0,
                offset_norm: float = 0.0) -> dict:
    """Return ``{'q','k','v','do'}`` as contiguous bf16 CPU tensors ``[B,H,N,d]``."""
    g = torch.Generator().manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if qkv_scale != 1.0:
        q.mul_(qkv_scale)
        k.mul_(qkv_scale)
        v.mul_(qkv_scale)
    if offset_norm > 0.0:
        gh = torch.randn((H, d), generator=g, dtype=torch.float32)
        u = offset_norm * gh / gh.norm(dim=-1, keepdim=True)
        q.add_(u.view(1, H, 1, d))
        k.add_(u.view(1, H, 1, d))
    return {n: t.to(torch.bfloat16).contiguous() for n, t in
            (("q", q), ("k", k), ("v", v), ("do", do))}


def workload_inputs(w: Workload) -> dict:
    """Dense workloads: ``{'q','k','v','do'}`` bf16 ``[B,H,N,d]``.  Variable-length
    workloads: the same keys as token-major bf16 ``[T, H, d]`` (T = sum of the
    lengths, drawn in the order Q, K, V, dO as fp32 randn of that shape) plus
    ``'cu_seqlens'``, int32 ``[B+1]`` offsets."""
    if w.lens:
        g = torch.Generator().manual_seed(int(w.seed))
        T = sum(w.lens)
        out = {n: torch.randn((T, w.H, w.d), generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()
               for n in ("q", "k", "v", "do")}
        cu = [0]
        for L in w.lens:
            cu.append(cu[-1] + L)
        out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32)
        return out
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.qkv_scale, w.offset_norm)


def block_mask(kind: str, H: int, N: int, seed: int = 0, block: int = 128) -> torch.Tensor:
    """Seeded synthetic block mask, uint8 ``[H, nt, nt]`` with ``nt = ceil(N / block)``.

    Structures of block-sparse attention patterns (the pages' section 3.2 on
    block-sparse attention names no specific pattern):
      * ``"random:<density>"`` -- each block kept with that probability,
        drawn per head;
      * ``"local:<w>,global:<g>"`` -- a band of ``w`` block diagonals on each
        side of the main one plus the first ``g`` block rows and columns (a
        sliding window with global tokens), the same for every head;
      * ``"ones"`` / ``"zeros"``.
    """
    nt = (N + block - 1) // block
    if kind == "ones":
        return torch.ones((H, nt, nt), dtype=torch.uint8)
    if kind == "zeros":
        return torch.zeros((H, nt, nt), dtype=torch.uint8)
    if kind.startswith("random:"):
        g = torch.Generator().manual_seed(int(seed))
        return (torch.rand((H, nt, nt), generator=g) < float(kind.split(":")[1])).to(torch.uint8)
    if kind.startswith("local:"):
        parts = dict(p.split(":") for p in kind.split(","))
        w, gl = int(parts["local"]), int(parts.get("global", 0))
        i = torch.arange(nt)
        m = ((i[:, None] - i[None, :]).abs() <= w) | (i[:, None] < gl) | (i[None, :] < gl)
        return m.to(torch.uint8).unsqueeze(0).expand(H, nt, nt).contiguous()
    raise ValueError(f"unknown block mask kind {kind!r}")


def visible_block_fraction(mask: torch.Tensor, causal: bool) -> float:
    """Work of a block mask relative to the dense non-causal problem, counting
    a diagonal block as half under the causal mask (the convention that makes
    dense causal attention half of dense)."""
    m = mask.to(torch.float64)
    nt = m.shape[-1]
    if causal:
        w = torch.tril(torch.ones(nt, nt, dtype=torch.float64), -1) + 0.5 * torch.eye(nt, dtype=torch.float64)
        m = m * w
    return float(m.sum() / (m.shape[0] * nt * nt))


def sample_rows(N: int, count: int, seed: int) -> list:
    """Sorted sample of ``count`` distinct rows of ``range(N)`` that always
    contains 0 and N-1, drawn from a generator seeded with ``1000 + seed``."""
    if count >= N:
        return list(range(N))
    g = torch.Generator().manual_seed(1000 + int(seed))
    perm = torch.randperm(N - 2, generator=g)[: max(0, count - 2)] + 1
    rows = sorted(set([0, N - 1] + perm.tolist()))
    return rows
