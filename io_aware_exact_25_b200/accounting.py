"""Work and traffic accounting for the attention path (bench reporting).

FLOPs follow the attention convention: 4*B*H*N^2*d for the forward (two
GEMMs of 2*N^2*d each), halved when causal, and 2.5x that for the backward.
Algorithmic bytes are what the fused kernels must move at the least: each
input read once and each output written once.  The standard-attention figures
are the pages' own accounting of a materialised score matrix ("FlashAttention
for Efficient Training", section 1.3, and Key Innovations: Tiling and
Recomputation) and are reported as context only.
"""
from __future__ import annotations


def score_matrix_bytes(B: int, H: int, N: int, bytes_per_elem: int = 4) -> int:
    """Bytes of one materialised N x N score matrix per head, all heads."""
    return int(bytes_per_elem) * B * H * N * N


def standard_attention_bandwidth(B: int, N: int, t_s: float) -> float:
    """Bandwidth (B/s) standard attention needs to write and re-read S and P
    (8 B N^2 bytes) within t_s seconds."""
    return 8.0 * B * N * N / t_s


def tiling_memory_saving(N: int, tile: int) -> int:
    """Factor by which keeping only a tile x tile block resident shrinks the
    score-matrix footprint: N^2 / tile^2."""
    return (N * N) // (tile * tile)


def fwd_bytes(B: int, H: int, N: int, d: int) -> int:
    """Read Q, K, V and write O (bf16), write lse (fp32)."""
    return 4 * B * H * N * d * 2 + 4 * B * H * N


def bwd_bytes(B: int, H: int, N: int, d: int) -> int:
    """Read Q, K, V, O, dO and write dQ, dK, dV (bf16); read lse, write and
    read D (fp32).  The fp32 dQ accumulator is scratch and is not counted."""
    return 8 * B * H * N * d * 2 + 3 * 4 * B * H * N


def fwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    f = 4.0 * B * H * N * N * d
    return f / 2.0 if causal else f


def bwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    return 2.5 * fwd_flops(B, H, N, d, causal)
