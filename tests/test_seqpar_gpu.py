"""The per-rank pieces of sequence parallelism (fa_fwd_partial,
fa_merge_partials, fa_weight_partial, fa_bwd_recompute_range) against the
fp64 oracle (GPU).

"FlashAttention for Efficient Training", section 5.3 (Sequence Parallelism
for Long Contexts).  One GPU plays every rank in turn: each key window gets
its own softmax piece and its own backward workspace; the pieces are either
stacked and merged or weighted and summed, and the windows' fp32 dQ
accumulators summed -- the data the NCCL all-gather and all-reduce of
io_aware_exact_25_b200.seqpar exchange (their bookkeeping is tested over
gloo in tests/test_seqpar_gloo.py; here torch sums stand in for the
all-reduce).  Every element is compared with the bar of tests/parity.py.
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


def _weighted_forward(x, windows, causal, scale, p, seed):
    """The summed exchange: every rank weights its own piece with all the
    pieces' lse, the weighted pieces are added (the all-reduce) and one
    one-piece merge converts the sum to bf16."""
    q = x["q"]
    parts = [binding.fwd_partial(q, x["k"][:, :, a:b].contiguous(), x["v"][:, :, a:b].contiguous(), a,
                                 causal=causal, scale=scale, dropout_p=p, seed=seed) for a, b in windows]
    all_lse = torch.stack([t[1] for t in parts]).contiguous()
    lse_w = None
    for r, (po, _) in enumerate(parts):
        _, lse_r = binding.weight_partial(po, all_lse, r)
        if lse_w is None:
            lse_w = lse_r
        else:
            assert torch.equal(lse_r, lse_w)  # every rank forms the same lse
    total = torch.stack([t[0] for t in parts]).sum(0)
    o, lse = binding.merge_partials(total.unsqueeze(0).contiguous(), lse_w.unsqueeze(0).contiguous())
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    return o, lse, parts


@pytest.mark.parametrize("N,d,causal,world,p", [
    (1000, 128, True, 2, 0.0), (1000, 64, False, 3, 0.0), (777, 128, True, 4, 0.1), (384, 64, True, 8, 0.0),
    (2048, 128, True, 5, 0.0)])
def test_weighted_pieces_sum_to_the_whole_problem(cuda_device, N, d, causal, world, p):
    B, H, seed = 1, 2, 23
    x = make_inputs(B, H, N, d, seed=N + world)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    scale = 1.0 / math.sqrt(d)
    windows = key_windows(N, world, causal)
    o, lse, parts = _weighted_forward(xd, windows, causal, scale, p, seed)
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=causal, p_drop=p, seed=seed)
    parity.check("O", o, ro)
    parity.check_lse(lse, rlse)
    # against the gather exchange: the same lse, O within one bf16 rounding
    xd2 = {n: t.to(cuda_device) for n, t in x.items()}
    parts2 = [binding.fwd_partial(xd2["q"], xd2["k"][:, :, a:b].contiguous(), xd2["v"][:, :, a:b].contiguous(), a,
                                  causal=causal, scale=scale, dropout_p=p, seed=seed) for a, b in windows]
    og, lseg = binding.merge_partials(torch.stack([t[0] for t in parts2]), torch.stack([t[1] for t in parts2]))
    torch.cuda.synchronize()
    assert (lse - lseg).abs().max().item() <= 1e-5
    assert ((o.float() - og.float()).abs() <= og.float().abs() * 2 ** -7 + 1e-6).all()


@pytest.mark.parametrize("d,S", [(64, 1), (128, 3), (64, 40), (128, 33)])
def test_weight_partial_against_its_definition(cuda_device, d, S):
    """Random pieces and logsumexps, some -inf and one row -inf in every
    piece, against the definition in fp64: lse = ln sum_s e^lse_s,
    piece * e^(lse_part - lse); 0 and lse = -inf where nothing is seen.
    S = 33 and 40 exceed the 32 lanes that share a row's reduction."""
    B, H, N = 2, 3, 130
    g = torch.Generator().manual_seed(d + S)
    all_lse = torch.randn((S, B, H, N), generator=g, dtype=torch.float64) * 6
    all_lse[torch.rand((S, B, H, N), generator=g) < 0.3] = float("-inf")
    all_lse[:, 1, 2, 7] = float("-inf")  # a row that no piece sees
    all_lse[:, 0, 0, 5] = 80.0  # equal pieces: lse = 80 + ln S
    pieces = torch.randn((S, B, H, N, d), generator=g, dtype=torch.float64)
    all_lse = all_lse.float().double()  # the values the kernel sees
    ref_lse = torch.logsumexp(all_lse, dim=0)
    lse_dev = all_lse.float().to(cuda_device).contiguous()
    for part in sorted({0, S // 2, S - 1}):
        po = pieces[part].float().to(cuda_device).contiguous()
        out, lse = binding.weight_partial(po, lse_dev, part)
        torch.cuda.synchronize()
        mine = all_lse[part]
        w = torch.where(torch.isneginf(mine), torch.zeros_like(mine), torch.exp(mine - ref_lse))
        w = torch.nan_to_num(w, nan=0.0)
        ref = pieces[part].float().double() * w[..., None]
        got = out.double().cpu()
        # fp32 arithmetic: lse rounded at |lse| <= 84 (half an ulp 3.8e-6) plus
        # the sum of up to 40 terms and logf, exp of the difference
        assert torch.allclose(got, ref, rtol=2e-5, atol=1e-30), (got - ref).abs().max().item()
        assert torch.equal(got[w == 0], torch.zeros_like(got[w == 0]))
        lc = lse.double().cpu()
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isneginf(lc), ~fin)
        assert ((lc[fin] - ref_lse[fin]).abs() <= 1e-5 + 1e-7 * ref_lse[fin].abs()).all()
        assert abs(lc[0, 0, 5].item() - (80 + math.log(S))) <= 1e-4


def test_one_rank_nccl_group_runs_the_cuda_orchestration(cuda_device, tmp_path):
    """seqpar.forward / seqpar.backward with the CUDA steps and real NCCL
    collectives over a one-rank group (no kernel waits on another rank):
    one window holds every key, so O, lse, dK and dV are the dense path's and
    every output meets the oracle, for both forward exchanges."""
    import torch.distributed as dist
    from datetime import timedelta
    from io_aware_exact_25_b200 import seqpar
    if dist.is_initialized():
        pytest.skip("a process group is already initialised in this process")
    B, H, N, d = 1, 2, 700, 128
    x = make_inputs(B, H, N, d, seed=77)
    xd = {n: t.to(cuda_device) for n, t in x.items()}
    o0, lse0 = binding.fwd(xd["q"], xd["k"], xd["v"], causal=True)
    dq0, dk0, dv0 = binding.bwd(xd["q"], xd["k"], xd["v"], o0, xd["do"], lse0, causal=True)
    scale = 1.0 / math.sqrt(d)
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=True)
    rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, causal=True)
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, causal=True)
    dist.init_process_group("nccl", init_method="file://" + str(tmp_path / "store"), rank=0, world_size=1,
                            timeout=timedelta(seconds=60))
    try:
        for exchange in ("sum", "gather"):
            o, lse = seqpar.forward(xd["q"], xd["k"], xd["v"], 0, causal=True, exchange=exchange)
            dq, dk, dv = seqpar.backward(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, 0, causal=True)
            torch.cuda.synchronize()
            assert binding.device_error() == 0
            assert (o.float() - o0.float()).abs().max().item() <= 2 ** -8, exchange
            assert (lse - lse0).abs().max().item() <= 1e-5, exchange
            assert torch.equal(dk, dk0) and torch.equal(dv, dv0), exchange
            assert (dq.float() - dq0.float()).abs().max().item() <= 2 ** -7, exchange
            parity.check("O", o, ro)
            parity.check_lse(lse, rlse)
            parity.check("dQ", dq, rdq)
            parity.check("dK", dk, rdk)
            parity.check("dV", dv, rdv)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,H,N,d,S", [(2, 3, 130, 64, 1), (2, 3, 130, 128, 3), (2, 3, 130, 64, 40),
                                        (2, 3, 130, 128, 8), (3, 2, 6667, 128, 3), (3, 5, 20500, 64, 2)])
def test_merge_partials_against_its_definition(cuda_device, B, H, N, d, S):
    """fa_merge_partials on random pieces and logsumexps, some -inf and one
    row -inf in every piece, against the definition in fp64: lse = ln sum_s
    e^lse_s, O = sum_s e^(lse_s - lse) O_s rounded to bf16; O = 0 and
    lse = -inf where nothing is seen.  The kernel's grid (1184 blocks of 8
    warps) takes rows in groups of G per warp, G the largest power of two up
    to 32 with G x 9472 <= rows: G = 1 for 780 rows, 4 for 40002 and 32 for
    307500 rows, the last two ending in a partial group."""
    g = torch.Generator().manual_seed(100 + d + S + N)
    all_lse = torch.randn((S, B, H, N), generator=g, dtype=torch.float64) * 6
    all_lse[torch.rand((S, B, H, N), generator=g) < 0.3] = float("-inf")
    all_lse[:, 0, 1, 9] = float("-inf")
    all_lse[0, 1, 1, 3] = 5.0  # one piece alone: O is that piece
    all_lse[1:, 1, 1, 3] = float("-inf")
    all_lse = all_lse.float().double()
    pieces = torch.randn((S, B, H, N, d), generator=g, dtype=torch.float64).float().double()
    o, lse = binding.merge_partials(pieces.float().to(cuda_device).contiguous(),
                                    all_lse.float().to(cuda_device).contiguous())
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    ref_lse = torch.logsumexp(all_lse, dim=0)
    w = torch.nan_to_num(torch.exp(all_lse - ref_lse), nan=0.0)
    ref = (w[..., None] * pieces).sum(0)
    got = o.double().cpu()
    # bf16 output: half an ulp (at most 2^-8 of |O|) plus the fp32 sum of up to
    # 40 weighted terms of magnitude < 5 (2e-5)
    assert ((got - ref).abs() <= ref.abs() * 2 ** -8 + 2e-5).all(), (got - ref).abs().max().item()
    assert torch.equal(got[0, 1, 9], torch.zeros(d, dtype=torch.float64))
    assert torch.equal(got[1, 1, 3], pieces[0, 1, 1, 3].float().bfloat16().double())
    lc = lse.double().cpu()
    fin = torch.isfinite(ref_lse)
    assert torch.equal(torch.isneginf(lc), ~fin)
    assert ((lc[fin] - ref_lse[fin]).abs() <= 1e-5 + 1e-7 * ref_lse[fin].abs()).all()
