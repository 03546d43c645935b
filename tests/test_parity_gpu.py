"""GPU parity: the sm_100a kernels (through the C ABI) against the fp64 oracle.

Tolerances (bf16 inputs and outputs, fp32 accumulation; tests/parity.py): for
O, dQ, dK, dV max |err| <= 2e-2 and relative L2 error <= 5e-3, with one
counted and reported exception for bf16 rounding at |ref| >= 4; lse within
1e-3; dropout keep masks bit-exact.  Small cases compare every element; the long-context
workloads compare sampled query rows (O, lse, dQ) and sampled key rows
(dK, dV) the oracle computes one by one, plus identities that hold at any
size.
"""
import math
import time

import numpy as np
import pytest
import torch

import oracle
import parity
from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import WORKLOADS, make_inputs, sample_rows, workload_inputs

pytestmark = pytest.mark.gpu

check = parity.check
check_lse = parity.check_lse


def _to(x, dev):
    return {n: t.to(dev) for n, t in x.items()}


def _run(xd, causal, scale, p=0.0, seed=0, backward=True):
    o, lse = binding.fwd(xd["q"], xd["k"], xd["v"], causal=causal, scale=scale, dropout_p=p, seed=seed)
    grads = None
    if backward:
        grads = binding.bwd(xd["q"], xd["k"], xd["v"], o, xd["do"], lse, causal=causal, scale=scale,
                            dropout_p=p, seed=seed)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    return o, lse, grads


def _full_compare(x, o, lse, grads, scale, causal, p=0.0, seed=0):
    B, H, N, d = x["q"].shape
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], scale, causal=causal, p_drop=p, seed=seed)
    check("O", o, ro)
    check_lse(lse, rlse)
    if grads is not None:
        dq, dk, dv = grads
        rdq, _, dev = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, causal=causal, p_drop=p, seed=seed)
        rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, causal=causal, p_drop=p, seed=seed)
        assert dev < 1e-9
        check("dQ", dq, rdq)
        check("dK", dk, rdk)
        check("dV", dv, rdv)


# ------------------------------------------------------------ small cases

@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload_all_elements(cuda_device, causal):
    w = WORKLOADS["tiny"]
    x = workload_inputs(w)
    o, lse, grads = _run(_to(x, cuda_device), causal, w.scale)
    _full_compare(x, o, lse, grads, w.scale, causal)


@pytest.mark.parametrize("N,d", [(1, 64), (77, 128), (129, 64), (300, 128), (640, 64), (1000, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_and_multi_tile_lengths(cuda_device, N, d, causal):
    """Lengths that are not a multiple of the 128-row tile, below one tile,
    and spanning several tiles with a ragged tail."""
    x = make_inputs(2, 3, N, d, seed=N + d)
    scale = 1.0 / math.sqrt(d)
    o, lse, grads = _run(_to(x, cuda_device), causal, scale)
    _full_compare(x, o, lse, grads, scale, causal)


@pytest.mark.parametrize("d", [64, 128])
def test_non_default_scale_and_peaked_rows(cuda_device, d):
    x = make_inputs(1, 4, 512, d, seed=21, offset_norm=2.0)
    scale = 0.7 / math.sqrt(d)
    for causal in (False, True):
        o, lse, grads = _run(_to(x, cuda_device), causal, scale)
        _full_compare(x, o, lse, grads, scale, causal)


def _rounding_model_bounds(x, scale, causal):
    """Per-element bounds on the dQ and dK errors that the backward's bf16
    operands account for, from fp64 values of the definition.

    The tensor cores take dS rounded to bf16 (half an ulp: a relative error of
    at most 2^-9 per element), and D_i = dO_i . O_i is formed from the stored
    bf16 O (an absolute error of at most 2^-9 sum_c |dO_ic O_ic|, which enters
    every dS_ij = P_ij (dP_ij - D_i) of the row).  Summed with absolute values,
    with twice that unit to cover the smaller terms (P kept as fp16 pairs, the
    fp32 sums):
        |err dQ_ic| <= 2e-2 + 2^-8 scale sum_j (|dS_ij| + P_ij a_i) |K_jc|
        |err dK_jc| <= 2e-2 + 2^-8 scale sum_i (|dS_ij| + P_ij a_i) |Q_ic|
    with a_i = sum_c |dO_ic O_ic|.  Returns ([BH, N, d], [BH, N, d]).
    """
    q, k, v, do = (x[n].to(torch.float64) for n in ("q", "k", "v", "do"))
    s = (q @ k.transpose(-1, -2)) * scale
    if causal:
        N = s.shape[-1]
        s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    p = torch.softmax(s, dim=-1)
    o = p @ v
    dp = do @ v.transpose(-1, -2)
    ds = p * (dp - (p * dp).sum(-1, keepdim=True))
    w = ds.abs() + p * (do * o).abs().sum(-1, keepdim=True)
    unit = 2.0 ** -8 * scale
    bq = parity.MAX_ABS + unit * (w @ k.abs())
    bk = parity.MAX_ABS + unit * (w.transpose(-1, -2) @ q.abs())
    B, H, N, d = q.shape
    return bq.reshape(B * H, N, d).numpy(), bk.reshape(B * H, N, d).numpy()


def test_large_score_range_triggers_rescaling(cuda_device):
    """Row maxima that grow across key tiles exercise the online rescaling
    of O and l (key norms rising from 0.2 to 6 along the sequence, scores
    spanning hundreds in base-2 units).  O, lse and dV meet the full bar.
    The keys, far larger here than in any workload, multiply the bf16
    rounding of dS in dQ = scale dS K (and the queries in dK): dQ and dK are
    held, element by element, to the bound that rounding accounts for
    (_rounding_model_bounds), and to the relative L2 bar."""
    g = torch.Generator().manual_seed(5)
    B, H, N, d = 1, 2, 768, 64
    q = torch.randn(B, H, N, d, generator=g)
    k = torch.randn(B, H, N, d, generator=g) * torch.linspace(0.2, 6.0, N).view(1, 1, N, 1)
    v = torch.randn(B, H, N, d, generator=g)
    do = torch.randn(B, H, N, d, generator=g)
    x = {n: t.to(torch.bfloat16).contiguous() for n, t in zip(("q", "k", "v", "do"), (q, k, v, do))}
    scale = 1.0 / math.sqrt(d)
    for causal in (False, True):
        o, lse, (dq, dk, dv) = _run(_to(x, cuda_device), causal, scale)
        _full_compare(x, o, lse, None, scale, causal)
        rdq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], scale, causal=causal)
        rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], scale, causal=causal)
        check("dV", dv, rdv)
        bq, bk = _rounding_model_bounds(x, scale, causal)
        for name, got, ref, bound in (("dQ", dq, rdq, bq), ("dK", dk, rdk, bk)):
            gv = got.float().cpu().numpy().astype(np.float64).reshape(ref.shape)
            err = np.abs(gv - ref)
            worst = np.unravel_index(np.argmax(err / bound), err.shape)
            print(f"rescaling causal={causal} {name}: max err {err.max():.3e}, max err/bound "
                  f"{(err / bound).max():.3f}, {int((err > parity.MAX_ABS).sum())} elements above 2e-2")
            assert np.all(err <= bound), (f"{name}: err {err[worst]:.3e} at {worst} above its rounding bound "
                                          f"{bound[worst]:.3e}")
            rel = np.linalg.norm(gv - ref) / np.linalg.norm(ref)
            assert rel <= parity.REL_L2, f"{name}: rel L2 {rel:.3e}"


@pytest.mark.parametrize("d", [64, 128])
def test_many_key_tiles_per_query_tile(cuda_device, d):
    """32 key tiles per query tile, non-causal, every element compared.  The
    forward's S_t(j) overwrites the tensor-memory columns that hold P_t(j-1)
    while the product reading P_t(j-1) is queued just before it, and the
    backward's S(i+1) overwrites P^T(i) behind dV(i): both rely on one
    thread's MMAs executing in issue order.  A long run of tiles with
    distinct values in every tile catches any overlap of the two."""
    B, H, N = 1, 2, 4096
    x = make_inputs(B, H, N, d, seed=600 + d)
    scale = 1.0 / math.sqrt(d)
    o, lse, grads = _run(_to(x, cuda_device), False, scale)
    _full_compare(x, o, lse, grads, scale, False)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_dropout_small_all_elements(cuda_device, d, causal):
    p, seed = 0.1, 4
    x = make_inputs(1, 2, 384, d, seed=31)
    scale = 1.0 / math.sqrt(d)
    o, lse, grads = _run(_to(x, cuda_device), causal, scale, p=p, seed=seed)
    _full_compare(x, o, lse, grads, scale, causal, p=p, seed=seed)


def test_dropout_mask_bit_exact(cuda_device):
    B, H, N = 2, 3, 1000
    heads = [0, 4, 5]
    rows = [0, 1, 17, 500, 999]
    for p, seed in ((0.1, 4), (0.5, 2 ** 40 + 7), (0.0, 1)):
        got = binding.dropout_mask(B, H, N, p, seed, heads, rows, device=cuda_device).cpu().numpy()
        ref = oracle.dropout_mask(B, H, N, p, seed, heads=heads, rows=rows)
        assert np.array_equal(got, ref)


def test_empty_problem_is_noop(cuda_device):
    q = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device=cuda_device)
    o, lse = binding.fwd(q, q, q, causal=True)
    assert o.shape == q.shape and lse.shape == (1, 2, 0)


@pytest.mark.parametrize("name", ["train2k", "train2k_causal"])
def test_training_shape_all_rows(cuda_device, name):
    w = WORKLOADS[name]
    x = workload_inputs(w)
    o, lse, grads = _run(_to(x, cuda_device), w.causal, w.scale)
    _full_compare(x, o, lse, grads, w.scale, w.causal)


# ------------------------------------------------- long-context workloads

def _sampled_compare(w, n_rows, kv_heads, kv_keys):
    x = workload_inputs(w)
    xd = _to(x, "cuda")
    o, lse, grads = _run(xd, w.causal, w.scale, p=w.p_drop, seed=w.seed)
    dq, dk, dv = grads
    BH = w.B * w.H
    rows = sample_rows(w.N, n_rows, w.seed)
    ro, rlse = oracle.forward(x["q"], x["k"], x["v"], w.scale, causal=w.causal, p_drop=w.p_drop, seed=w.seed,
                              rows=rows)
    ridx = torch.as_tensor(rows, device="cuda")
    check("O rows", o.view(BH, w.N, w.d)[:, ridx], ro)
    check_lse(lse.view(BH, w.N)[:, ridx], rlse)
    rdq, _, dev = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], w.scale, causal=w.causal, p_drop=w.p_drop,
                                    seed=w.seed, rows=rows)
    assert dev < 1e-9
    # causal row 0 sees one key, so its exact dQ is 0: D_0 = dO_0 . O_0 then
    # carries the bf16 rounding of O_0 straight into dQ_0 (only the absolute
    # bound is meaningful for it)
    check("dQ rows", dq.view(BH, w.N, w.d)[:, ridx], rdq, exclude_rows=[0] if w.causal else None)
    t0 = time.perf_counter()
    rdk, rdv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], w.scale, causal=w.causal, p_drop=w.p_drop,
                                  seed=w.seed, heads=kv_heads, keys=kv_keys)
    print(f"{w.name}: oracle dK/dV for {len(kv_keys)} keys x {len(kv_heads)} heads from key {min(kv_keys)}: "
          f"{time.perf_counter() - t0:.1f} s on {oracle.num_threads()} threads")
    hidx = torch.as_tensor(kv_heads, device="cuda")
    kidx = torch.as_tensor(kv_keys, device="cuda")
    check("dK rows", dk.view(BH, w.N, w.d)[hidx][:, kidx], rdk)
    check("dV rows", dv.view(BH, w.N, w.d)[hidx][:, kidx], rdv)
    # identities over every head and key (any size): sum_j dK_j = 0 and, without
    # dropout, sum_j dV_j = sum_i dO_i; both in fp32 sums of bf16 outputs
    sdk = dk.float().sum(dim=2)
    scale_dk = dk.float().abs().sum(dim=2)
    assert (sdk.abs() <= 1e-2 * scale_dk + 1e-2).all()
    if w.p_drop == 0.0:
        sdv = dv.float().sum(dim=2)
        sdo = xd["do"].float().sum(dim=2)
        assert ((sdv - sdo).abs() <= 1e-2 * dv.float().abs().sum(dim=2) + 1e-2).all()
    if w.p_drop > 0.0:
        mrows = rows[:16]
        got = binding.dropout_mask(w.B, w.H, w.N, w.p_drop, w.seed, list(range(BH)), mrows).cpu().numpy()
        ref = oracle.dropout_mask(w.B, w.H, w.N, w.p_drop, w.seed, rows=mrows)
        assert np.array_equal(got, ref)


def test_long8k_causal_sampled(cuda_device):
    w = WORKLOADS["long8k_causal"]
    keys = sample_rows(w.N, 64, w.seed + 100)
    _sampled_compare(w, 512, kv_heads=[0, w.B * w.H - 1], kv_keys=keys)


# Keys near j = 0 are seen by every causal query tile: they carry the longest
# dK/dV accumulation and the persistent grid's heaviest work items, so both
# long workloads check them along with keys spread over the whole sequence.
# The oracle needs the row statistics of every query that sees a checked key,
# an O(N^2 d) pass per head from key 0 on.
def _early_and_spread_keys(N, seed, n_spread):
    early = [0, 1, 2, 63, 64, 127, 128, 129, 255, 1000, 2047]
    return sorted(set(early + sample_rows(N, n_spread, seed + 200)))


def test_long32k_causal_sampled(cuda_device):
    w = WORKLOADS["long32k_causal"]
    keys = _early_and_spread_keys(w.N, w.seed, 48)
    _sampled_compare(w, 256, kv_heads=[0, w.H - 1], kv_keys=keys)


def test_long64k_causal_dropout_sampled(cuda_device):
    w = WORKLOADS["long64k_causal_dropout"]
    keys = _early_and_spread_keys(w.N, w.seed, 32)
    _sampled_compare(w, 128, kv_heads=[0, 5], kv_keys=keys)


def test_backward_stages_equal_one_call(cuda_device):
    """fa_bwd_prepare + fa_bwd_recompute + fa_bwd_finalize is fa_bwd."""
    x = _to(make_inputs(2, 2, 640, 128, seed=41), cuda_device)
    o, lse = binding.fwd(x["q"], x["k"], x["v"], causal=True)
    a = binding.bwd(x["q"], x["k"], x["v"], o, x["do"], lse, causal=True)
    b = binding.bwd_stages(x["q"], x["k"], x["v"], o, x["do"], lse, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])  # dK, dV: no atomics
    assert (a[0].float() - b[0].float()).abs().max().item() <= 2 ** -7  # dQ: atomic order
