"""Every entry point through the bounds-checking build (libfa_sm100_debug.so,
compiled with FA_DEBUG) on small cases.

In that build each global-memory access the kernels derive from their work
decomposition is checked against the extent the call's shape and strides
give its buffer (csrc/debug_check.cuh).  A case passes when no check failed
(device error 0, an empty record) and the results equal the release build's:
bit for bit for O, lse, dK and dV (their summation order is fixed), and to
within the fp32 accumulation order for dQ, whose partials are added in a
run-dependent order.  The cases cover ragged lengths, both head dimensions,
causal and not, strided (BSHD) tensors, split-KV, block-sparse masks,
variable-length batches with padded slots, dropout, the key windows of
sequence parallelism and the no-allocation backward.
"""
import math

import pytest
import torch

from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import block_mask, make_inputs

pytestmark = pytest.mark.gpu


def _run_both(fn):
    """fn() with the release build, then with the bounds-checking build;
    asserts that no check failed in the latter."""
    ref = fn()
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    with binding.use_library(binding.DEBUG_LIB_PATH) as lib:
        assert lib.fa_debug_build() == 1
        binding.debug_bounds_record()  # start from an empty record
        got = fn()
        torch.cuda.synchronize()
        rec = binding.debug_bounds_record()
        err = binding.device_error()
    assert rec[0] == 0, f"bounds check failed: site {rec[1]}, offset {rec[2]}, limit {rec[3]}, block {rec[4]}, " \
                        f"thread {rec[5]} ({rec[0]} failures)"
    assert err == 0, f"device error {err}"
    return ref, got


def _same(ref, got, names, dq_names=()):
    for n, r, g in zip(names, ref, got):
        if n in dq_names:
            assert (r.float() - g.float()).abs().max().item() <= 2 ** -6, n
        else:
            assert torch.equal(r, g), n


def _dev(x, dev):
    return {n: t.to(dev) for n, t in x.items()}


@pytest.mark.parametrize("N,d,causal,p", [(777, 64, True, 0.0), (384, 128, False, 0.0), (1000, 128, True, 0.1),
                                          (300, 64, False, 0.2)])
def test_dense(cuda_device, N, d, causal, p):
    x = _dev(make_inputs(2, 3, N, d, seed=N), cuda_device)

    def run():
        o, lse = binding.fwd(x["q"], x["k"], x["v"], causal=causal, dropout_p=p, seed=3)
        dq, dk, dv = binding.bwd(x["q"], x["k"], x["v"], o, x["do"], lse, causal=causal, dropout_p=p, seed=3)
        return o, lse, dq, dk, dv

    ref, got = _run_both(run)
    _same(ref, got, ("o", "lse", "dq", "dk", "dv"), ("dq",))


def test_strided_bshd(cuda_device):
    B, H, N, d = 2, 4, 520, 128
    x = make_inputs(B, H, N, d, seed=9)
    # [B, N, H, d] storage viewed as [B, H, N, d]
    t = {n: v.transpose(1, 2).contiguous().to(cuda_device).transpose(1, 2) for n, v in x.items()}

    def run():
        o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=cuda_device).transpose(1, 2)
        o, lse = binding.fwd(t["q"], t["k"], t["v"], causal=True, o=o)
        dq = torch.empty_like(o)
        dk = torch.empty_like(o)
        dv = torch.empty_like(o)
        binding.bwd(t["q"], t["k"], t["v"], o, t["do"], lse, causal=True, dq=dq, dk=dk, dv=dv)
        return o, lse, dq, dk, dv

    ref, got = _run_both(run)
    _same(ref, got, ("o", "lse", "dq", "dk", "dv"), ("dq",))


def test_splitkv(cuda_device):
    x = _dev(make_inputs(1, 1, 4000, 128, seed=4), cuda_device)
    ref, got = _run_both(lambda: binding.fwd_splitkv(x["q"], x["k"], x["v"], causal=False, num_splits=5))
    # the merge's order is fixed as well
    _same(ref, got, ("o", "lse"))


@pytest.mark.parametrize("kind,causal", [("local:2,global:1", True), ("random:0.3", False)])
def test_blocksparse(cuda_device, kind, causal):
    B, H, N, d = 1, 2, 900, 64
    x = _dev(make_inputs(B, H, N, d, seed=12), cuda_device)
    m = block_mask(kind, H, N, seed=5).to(cuda_device)

    def run():
        o, lse = binding.fwd(x["q"], x["k"], x["v"], causal=causal, block_mask=m)
        dq, dk, dv = binding.bwd(x["q"], x["k"], x["v"], o, x["do"], lse, causal=causal, block_mask=m)
        return o, lse, dq, dk, dv

    ref, got = _run_both(run)
    _same(ref, got, ("o", "lse", "dq", "dk", "dv"), ("dq",))


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_with_padded_slots(cuda_device, d):
    lens = [300, 1, 128, 0, 513]
    slot = 600
    H = 2
    g = torch.Generator().manual_seed(d)
    T = slot * len(lens)
    tok = {n: (torch.randn((T, H, d), generator=g) * 0.5).to(torch.bfloat16).to(cuda_device)
           for n in ("q", "k", "v", "do")}
    cu = torch.arange(0, T + 1, slot, dtype=torch.int32, device=cuda_device)
    used = torch.tensor(lens, dtype=torch.int32, device=cuda_device)

    def run():
        o, lse = binding.fwd_varlen(tok["q"], tok["k"], tok["v"], cu, slot, seqused=used, causal=True)
        dq, dk, dv = binding.bwd_varlen(tok["q"], tok["k"], tok["v"], o, tok["do"], lse, cu, slot, seqused=used,
                                        causal=True)
        return o, lse, dq, dk, dv

    ref, got = _run_both(run)
    _same(ref, got, ("o", "lse", "dq", "dk", "dv"), ("dq",))


def test_sequence_parallel_pieces(cuda_device):
    """fa_fwd_partial, fa_merge_partials, fa_weight_partial and
    fa_bwd_recompute_range over three key windows, one of them ragged."""
    B, H, N, d = 1, 2, 700, 128
    x = _dev(make_inputs(B, H, N, d, seed=21), cuda_device)
    windows = [(0, 256), (256, 512), (512, N)]

    def run():
        parts = [binding.fwd_partial(x["q"], x["k"][:, :, a:b].contiguous(), x["v"][:, :, a:b].contiguous(), a,
                                     causal=True) for a, b in windows]
        o, lse = binding.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
        all_lse = torch.stack([p[1] for p in parts]).contiguous()
        weighted = [binding.weight_partial(p[0].clone(), all_lse, r)[0] for r, p in enumerate(parts)]
        out = [o, lse] + weighted
        for a, b in windows:
            ws = torch.empty(binding.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=cuda_device)
            binding.bwd_prepare(o, x["do"], lse, ws)
            dk, dv = binding.bwd_recompute_range(x["q"], x["k"][:, :, a:b].contiguous(),
                                                 x["v"][:, :, a:b].contiguous(), x["do"], a, ws, causal=True)
            out += [dk, dv]
        return out

    ref, got = _run_both(run)
    _same(ref, got, ["o", "lse"] + [f"w{r}" for r in range(3)] + [f"{n}{w}" for w in range(3) for n in ("dk", "dv")])


def test_noalloc_backward(cuda_device):
    B, H, N, d = 1, 2, 640, 64
    x = _dev(make_inputs(B, H, N, d, seed=30), cuda_device)
    o, lse = binding.fwd(x["q"], x["k"], x["v"], causal=True)

    def run():
        dq, dk, dv = (torch.empty_like(x["q"]) for _ in range(3))
        binding.bwd_noalloc(x["q"], x["k"], x["v"], o, x["do"], lse, dq, dk, dv, causal=True)
        return dq, dk, dv

    ref, got = _run_both(run)
    _same(ref, got, ("dq", "dk", "dv"), ("dq",))
    assert math.isfinite(float(got[0].float().sum()))
