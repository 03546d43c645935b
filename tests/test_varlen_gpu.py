"""Variable-length batches (fa_fwd_varlen / fa_bwd_varlen) against the fp64
oracle (GPU).

"FlashAttention for Efficient Training" section 5.2 (Handling Variable
Sequence Lengths, Efficient Padding and Masking): a score is -inf unless its
key lies within the sequence, and no work is spent on padded tokens.  The
oracle takes the padded [B, H, N, d] layout with per-batch lengths; the
kernels take the token-major (batch, seq_len, num_heads, head_dim) layout
with offsets, either packed (slots exactly the sequences) or padded (slots
of N tokens, the first L_b real).  Every element is compared, with the bar
of tests/parity.py; padding rows must be exactly O = 0, lse = -inf and
dQ = dK = dV = 0.
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


def _padded_inputs(lens, H, d, seed, pad_value_seed=None):
    """Oracle-layout inputs [B, H, N, d] with N = max(lens); the padding rows
    hold large random values (never zeros), which must not reach any result."""
    B, N = len(lens), max(max(lens), 1)
    x = make_inputs(B, H, N, d, seed=seed)
    g = torch.Generator().manual_seed(pad_value_seed if pad_value_seed is not None else seed + 1)
    for b, L in enumerate(lens):
        for n in x:
            x[n][b, :, L:] = (torch.randn(H, N - L, d, generator=g) * 8).to(torch.bfloat16)
    return x


def _pack(t, lens):
    """[B, H, N, d] -> token-major [sum(lens), H, d] holding the real rows only."""
    return torch.cat([t[b, :, :L].transpose(0, 1) for b, L in enumerate(lens)], dim=0).contiguous()


def _unpack(t, lens, N, fill=0.0):
    """Token-major [T, H, d] (packed) -> [B, H, N, d] with `fill` in the padding."""
    B, H, d = len(lens), t.shape[1], t.shape[2]
    out = torch.full((B, H, N, d), fill, dtype=t.dtype, device=t.device)
    off = 0
    for b, L in enumerate(lens):
        out[b, :, :L] = t[off:off + L].transpose(0, 1)
        off += L
    return out


def _oracle_all(x, lens, scale, causal, p=0.0, seed=0):
    kw = dict(causal=causal, p_drop=p, seed=seed, seqlens=lens)
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, **kw)
    rdq, _, dev = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, **kw)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, **kw)
    assert dev < 1e-9
    return ro, rlse, rdq, rdk, rdv


def _compare(lens, H, N, d, out, ref, causal, p):
    """out: padded-layout GPU results (o, lse [B,H,N], dq, dk, dv) as torch;
    ref: the oracle's, [B*H, N, ...]."""
    o, lse, dq, dk, dv = out
    ro, rlse, rdq, rdk, rdv = ref
    B = len(lens)
    real = np.zeros((B, N), bool)
    for b, L in enumerate(lens):
        real[b, :L] = True
    rmask = np.repeat(real, H, axis=0)  # [B*H, N]
    g = lambda t: t.detach().float().cpu().numpy().astype(np.float64).reshape(B * H, N, -1)
    # padding rows: exact zeros / -inf
    for name, t in (("O", o), ("dQ", dq), ("dK", dk), ("dV", dv)):
        assert np.all(g(t)[~rmask] == 0.0), f"{name}: padding rows not zero"
    assert np.all(np.isneginf(lse.detach().cpu().numpy().reshape(B * H, N)[~rmask])), "lse: padding rows"
    if not rmask.any():
        return
    idx = np.nonzero(rmask)
    for name, t, r in (("O", o, ro), ("dQ", dq, rdq), ("dK", dk, rdk), ("dV", dv, rdv)):
        got = torch.from_numpy(g(t)[idx])
        if name == "dQ" and causal and p > 0:
            # causal row 0 of each sequence sees one key: its exact dQ is 0 and
            # the bf16 rounding of the stored O_0 enters D_0 (relative error
            # undefined there; the absolute bound still applies)
            first = np.array([i == 0 for i in idx[1]])
            parity.check(name, got[first], r[idx][first])
            got, r_sel = got[~first], r[idx][~first]
            parity.check(name, got[None], r_sel[None])
            continue
        parity.check(name, got[None], r[idx][None])
    parity.check_lse(torch.from_numpy(lse.detach().cpu().numpy().reshape(B * H, N)[idx]), rlse[idx])


def _run_packed(x, lens, H, d, scale, causal, p=0.0, seed=0, dev="cuda"):
    N = x["q"].shape[2]
    packed = {n: _pack(t, lens).to(dev) for n, t in x.items()}
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=dev)
    maxs = max(max(lens), 1)
    o, lse = binding.fwd_varlen(packed["q"], packed["k"], packed["v"], cu, maxs, causal=causal, scale=scale,
                                dropout_p=p, seed=seed)
    dq, dk, dv = binding.bwd_varlen(packed["q"], packed["k"], packed["v"], o, packed["do"], lse, cu, maxs,
                                    causal=causal, scale=scale, dropout_p=p, seed=seed)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    T = sum(lens)
    lse_tok = lse.transpose(0, 1).reshape(T, H, 1)  # [H, T] -> [T, H, 1]
    outs = [_unpack(t, lens, N) for t in (o, dq, dk, dv)]
    lse_p = _unpack(lse_tok, lens, N, fill=float("-inf"))[..., 0]
    return outs[0], lse_p, outs[1], outs[2], outs[3]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_packed_mixed_lengths_all_elements(cuda_device, d, causal):
    """Lengths below one tile, not a multiple of 128, exactly one tile, and
    several tiles with a ragged tail, packed back to back."""
    lens = [300, 1, 128, 77, 513, 0, 200]
    H = 2
    x = _padded_inputs(lens, H, d, seed=700 + d)
    scale = 1.0 / math.sqrt(d)
    out = _run_packed(x, lens, H, d, scale, causal)
    _compare(lens, H, max(lens), d, out, _oracle_all(x, lens, scale, causal), causal, 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_packed_with_dropout(cuda_device, causal):
    lens = [384, 129, 250]
    H, d, p, seed = 2, 64, 0.1, 17
    x = _padded_inputs(lens, H, d, seed=711)
    scale = 1.0 / math.sqrt(d)
    out = _run_packed(x, lens, H, d, scale, causal, p=p, seed=seed)
    _compare(lens, H, max(lens), d, out, _oracle_all(x, lens, scale, causal, p=p, seed=seed), causal, p)


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_padded_slots_with_seqused(cuda_device, d, causal):
    """The pages' (batch, seq_len, num_heads, head_dim) padded batch: slots of
    N tokens, the first L_b real (seqused).  Padding tokens hold large random
    values; they must not reach any result, and their output rows must be
    zero (lse -inf)."""
    lens = [640, 100, 0, 333]
    B, H, N = len(lens), 3, 640
    x = _padded_inputs(lens, H, d, seed=720 + d)
    scale = 1.0 / math.sqrt(d)
    bshd = {n: t.transpose(1, 2).contiguous().to(cuda_device) for n, t in x.items()}  # [B, N, H, d]
    tok = {n: t.view(B * N, H, d) for n, t in bshd.items()}
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device=cuda_device)
    used = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    o = torch.full_like(tok["q"], 7.0)  # every output row is written: real or padding
    lse = torch.full((H, B * N), 7.0, dtype=torch.float32, device=cuda_device)
    binding.fwd_varlen(tok["q"], tok["k"], tok["v"], cu, N, seqused=used, causal=causal, scale=scale, o=o, lse=lse)
    grads = [torch.full_like(tok["q"], 7.0) for _ in range(3)]
    binding.bwd_varlen(tok["q"], tok["k"], tok["v"], o, tok["do"], lse, cu, N, seqused=used, causal=causal,
                       scale=scale, dq=grads[0], dk=grads[1], dv=grads[2])
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    to_bhnd = lambda t: t.view(B, N, H, d).transpose(1, 2)
    lse_p = lse.view(H, B, N).transpose(0, 1)
    out = (to_bhnd(o), lse_p, to_bhnd(grads[0]), to_bhnd(grads[1]), to_bhnd(grads[2]))
    _compare(lens, H, N, d, out, _oracle_all(x, lens, scale, causal), causal, 0.0)


def test_long_mixed_lengths(cuda_device):
    """Sequences of several thousand tokens next to short ones (d = 128,
    causal), every element compared."""
    lens = [4096, 1000, 2500, 64]
    H, d = 2, 128
    x = _padded_inputs(lens, H, d, seed=730)
    scale = 1.0 / math.sqrt(d)
    out = _run_packed(x, lens, H, d, scale, True)
    _compare(lens, H, max(lens), d, out, _oracle_all(x, lens, scale, True), True, 0.0)


def test_equal_lengths_match_the_dense_kernels(cuda_device):
    """B sequences of one length N packed back to back give the dense result:
    O and lse bit for bit, dK and dV bit for bit (deterministic), dQ within
    the rounding of its reduction order."""
    B, H, N, d = 3, 2, 777, 128
    x = {n: t.to(cuda_device) for n, t in make_inputs(B, H, N, d, seed=740).items()}
    lens = [N] * B
    o_d, lse_d = binding.fwd(x["q"], x["k"], x["v"], causal=True)
    g_d = binding.bwd(x["q"], x["k"], x["v"], o_d, x["do"], lse_d, causal=True)
    packed = {n: _pack(t, lens) for n, t in x.items()}
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device=cuda_device)
    o_v, lse_v = binding.fwd_varlen(packed["q"], packed["k"], packed["v"], cu, N, causal=True)
    g_v = binding.bwd_varlen(packed["q"], packed["k"], packed["v"], o_v, packed["do"], lse_v, cu, N, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(_pack(o_d, lens), o_v)
    assert torch.equal(lse_d.permute(1, 0, 2).reshape(H, B * N), lse_v)
    assert torch.equal(_pack(g_d[1], lens), g_v[1]) and torch.equal(_pack(g_d[2], lens), g_v[2])
    assert (_pack(g_d[0], lens).float() - g_v[0].float()).abs().max().item() <= 2 ** -7


def test_out_of_range_offsets_are_clamped_and_reported(cuda_device):
    """Offsets past the tensors are clamped (no access leaves them) and
    reported as device error 3; the call itself succeeds."""
    T, H, d = 300, 2, 64
    q = torch.randn(T, H, d, device=cuda_device).to(torch.bfloat16)
    cu = torch.tensor([0, 200, 500], dtype=torch.int32, device=cuda_device)  # 500 > T
    o = torch.zeros_like(q)
    lse = torch.zeros(H, T, device=cuda_device)
    binding.fwd_varlen(q, q, q, cu, 512, o=o, lse=lse)
    assert binding.device_error() == 3
    assert binding.device_error() == 0
    assert torch.isfinite(o.float()).all()
