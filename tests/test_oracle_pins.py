"""Pins for the fp64 CPU oracle (no GPU).

Each test ties the oracle to something other than itself: a closed form, an
invariant the mathematics fixes, central finite differences, torch's fp64
CPU ``scaled_dot_product_attention`` / autograd (a library special case), or
published constants.  A dropped term, a wrong sign or index, or a transposed
operand in the oracle fails at least one of them.

Passages: the attention definition and the numerically stable softmax
("FlashAttention for Efficient Training", sections 1 and 6.2), the logsumexp
statistic (section 3.2), dV = P^T dO (section 3.2, Integration with Autograd
Engines), causal masking (section 5.1), dropout fused after the softmax
(section 3, Fused Kernel Design).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_25_b200.inputs import make_inputs, sample_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).contiguous()


def _f64(t):
    return t.to(torch.float64)


def _torch_sdpa(q, k, v, scale, causal):
    return torch.nn.functional.scaled_dot_product_attention(
        _f64(q), _f64(k), _f64(v), is_causal=causal, scale=scale)


# ------------------------------------------------------------ hash pins

def test_hash_constants_match_published_values():
    ref = json.load(open(os.path.join(GOLDEN, "hash_constants.json")))
    c1, c2, g = oracle.hash_constants()
    assert c1 == int(ref["C1"]["value_hex"], 16)
    assert c2 == int(ref["C2"]["value_hex"], 16)
    assert g == int(ref["G"]["value_hex"], 16)
    # multipliers of an invertible mixer must be odd
    assert c1 % 2 == 1 and c2 % 2 == 1 and g % 2 == 1


def test_keep_threshold_closed_forms():
    assert oracle.keep_threshold(0.0) == 0
    assert oracle.keep_threshold(0.5) == 2 ** 15
    # ceil(0.1 * 2^16) = ceil(6553.6)
    assert oracle.keep_threshold(0.1) == 6554
    assert oracle.keep_threshold(0.25) == 2 ** 14
    # the largest p below 1 keeps nothing: T = 2^16 exceeds every 16-bit half
    assert oracle.keep_threshold(1.0 - 2.0 ** -20) == 2 ** 16


def test_adjacent_keys_use_independent_halves():
    """Keys 2u and 2u+1 of a row share one 32-bit mix but read disjoint
    halves of it: their keep decisions must be uncorrelated (a mask that
    read the same half, or the same bits, for both would make them equal),
    and the pair's keep rate must be (1 - p)^2."""
    p = 0.3
    mask = oracle.dropout_mask(1, 2, 1024, p, seed=8).astype(np.float64)
    even, odd = mask[..., 0::2].ravel(), mask[..., 1::2].ravel()
    n = even.size
    corr = np.corrcoef(even, odd)[0, 1]
    assert abs(corr) < 5 / math.sqrt(n)
    both = (even * odd).mean()
    assert abs(both - (1 - p) ** 2) < 5 * math.sqrt((1 - p) ** 2 * (1 - (1 - p) ** 2) / n)
    # and every key's rate on its own is 1 - p
    for half in (even, odd):
        assert abs(half.mean() - (1 - p)) < 5 * math.sqrt(p * (1 - p) / n)


def test_dropout_mask_statistics():
    p = 0.1
    B, H, N = 1, 2, 2048
    mask = oracle.dropout_mask(B, H, N, p, seed=4).astype(np.float64)
    n = mask.size
    keep = mask.mean()
    sigma = math.sqrt(p * (1 - p) / n)
    assert abs(keep - (1 - p)) < 5 * sigma
    # per-row and per-column keep rates
    row_rate = mask.mean(axis=2)
    col_rate = mask.mean(axis=1)
    s_line = math.sqrt(p * (1 - p) / N)
    assert np.all(np.abs(row_rate - (1 - p)) < 6 * s_line)
    assert np.all(np.abs(col_rate - (1 - p)) < 6 * s_line)
    # different seeds give different masks, same seed the same mask
    m2 = oracle.dropout_mask(B, H, N, p, seed=5)
    assert (m2.astype(np.float64) != mask).mean() > 0.1
    assert np.array_equal(oracle.dropout_mask(B, H, N, p, seed=4), mask.astype(np.uint8))


def test_hash_output_bits_balanced():
    vals = np.array([oracle.hash32(4, 0, h, i, j)
                     for h in range(2) for i in range(0, 64, 3) for j in range(128)], dtype=np.uint64)
    n = vals.size
    for bit in range(32):
        frac = ((vals >> np.uint64(bit)) & np.uint64(1)).mean()
        assert abs(frac - 0.5) < 5 * math.sqrt(0.25 / n), bit
    # every coordinate of the counter reaches the output
    base = oracle.hash32(7, 1, 2, 3, 4)
    for args in [(8, 1, 2, 3, 4), (7 + (1 << 32), 1, 2, 3, 4), (7, 0, 2, 3, 4), (7, 1, 3, 3, 4),
                 (7, 1, 2, 2, 4), (7, 1, 2, 3, 5)]:
        assert oracle.hash32(*args) != base


# --------------------------------------------------------- forward pins

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("scale", [None, 0.3])
def test_forward_matches_torch_fp64_sdpa(causal, scale):
    x = make_inputs(2, 3, 40, 16, seed=11)
    sc = 1 / math.sqrt(16) if scale is None else scale
    o, lse = oracle.forward(x["q"], x["k"], x["v"], sc, causal=causal)
    ref = _torch_sdpa(x["q"], x["k"], x["v"], sc, causal).reshape(6, 40, 16)
    assert np.max(np.abs(o - ref.numpy())) < 1e-12
    s = sc * _f64(x["q"]) @ _f64(x["k"]).transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(40, 40, dtype=torch.bool).triu(1), -math.inf)
    ref_lse = torch.logsumexp(s, dim=-1).reshape(6, 40)
    assert np.max(np.abs(lse - ref_lse.numpy())) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_visible_values(causal):
    B, H, N, d = 1, 1, 24, 8
    x = make_inputs(B, H, N, d, seed=3)
    k = x["k"][:, :, :1, :].expand(B, H, N, d).contiguous()  # every key equal
    sc = 0.5
    o, lse = oracle.forward(x["q"], k, x["v"], sc, causal=causal)
    v = _f64(x["v"])[0, 0]
    q = _f64(x["q"])[0, 0]
    k0 = _f64(k)[0, 0, 0]
    for i in range(N):
        n_vis = i + 1 if causal else N
        expect = v[:n_vis].mean(dim=0).numpy()
        assert np.max(np.abs(o[0, i] - expect)) < 1e-13
        s = sc * float(q[i] @ k0)
        assert abs(lse[0, i] - (s + math.log(n_vis))) < 1e-13


def test_one_hot_dominant_score_selects_one_value_row():
    B, H, N, d = 1, 1, 32, 8
    x = make_inputs(B, H, N, d, seed=5)
    q = torch.zeros(B, H, N, d)
    q[..., 0] = 8.0
    k = torch.zeros(B, H, N, d)
    jstar = 17
    k[0, 0, jstar, 0] = 8.0  # s = 64 for j*, 0 elsewhere (scale 1)
    o, lse = oracle.forward(_bf16(q), _bf16(k), x["v"], 1.0, causal=False)
    vj = _f64(x["v"])[0, 0, jstar].numpy()
    assert np.max(np.abs(o[0] - vj[None, :])) < 1e-20 + 40 * math.exp(-64) * 4
    assert np.max(np.abs(lse[0] - 64.0)) < 1e-12


def test_causal_row_zero_is_first_value_row():
    x = make_inputs(1, 2, 64, 16, seed=6)
    sc = 0.25
    o, lse = oracle.forward(x["q"], x["k"], x["v"], sc, causal=True)
    v = _f64(x["v"]).reshape(2, 64, 16)
    q = _f64(x["q"]).reshape(2, 64, 16)
    k = _f64(x["k"]).reshape(2, 64, 16)
    for h in range(2):
        assert np.array_equal(o[h, 0], v[h, 0].numpy())
        assert abs(lse[h, 0] - sc * float(q[h, 0] @ k[h, 0])) < 1e-14


@pytest.mark.parametrize("p_drop", [0.0, 0.1])
def test_probability_rows_sum_to_one(p_drop):
    # with V = 1 every output element is sum_j P_ij (no dropout)
    x = make_inputs(1, 2, 48, 8, seed=7)
    ones = torch.ones(1, 2, 48, 8, dtype=torch.bfloat16)
    for causal in (False, True):
        o, _ = oracle.forward(x["q"], x["k"], ones, 0.35, causal=causal)
        assert np.max(np.abs(o - 1.0)) < 1e-13
    if p_drop:
        # with dropout the row sums are sum_j P_ij Z_ij / (1 - p), whose mean is 1
        o, _ = oracle.forward(x["q"], x["k"], ones, 0.35, p_drop=p_drop, seed=9)
        assert np.max(o) > 1.0 or np.min(o) < 1.0


def test_linearity_and_permutation_equivariance():
    x = make_inputs(1, 1, 32, 8, seed=8)
    sc = 0.35
    o, _ = oracle.forward(x["q"], x["k"], x["v"], sc)
    o2, _ = oracle.forward(x["q"], x["k"], (2 * x["v"].float()).to(torch.bfloat16), sc)
    assert np.max(np.abs(o2 - 2 * o)) < 1e-13
    perm = torch.randperm(32, generator=torch.Generator().manual_seed(1))
    # permuting the query rows permutes the output rows
    op, _ = oracle.forward(x["q"][:, :, perm].contiguous(), x["k"], x["v"], sc)
    assert np.max(np.abs(op[0] - o[0][perm.numpy()])) < 1e-13
    # permuting keys and values together leaves the output unchanged
    ok, _ = oracle.forward(x["q"], x["k"][:, :, perm].contiguous(), x["v"][:, :, perm].contiguous(), sc)
    assert np.max(np.abs(ok - o)) < 1e-13


def test_shift_invariance_of_keys():
    g = torch.Generator().manual_seed(2)
    q = torch.randint(-3, 4, (1, 1, 20, 8), generator=g).float()
    k = torch.randint(-3, 4, (1, 1, 20, 8), generator=g).float()
    v = torch.randn(1, 1, 20, 8, generator=g)
    c = torch.randint(-2, 3, (8,), generator=g).float()  # integer shift: exact in bf16
    o, lse = oracle.forward(_bf16(q), _bf16(k), _bf16(v), 0.25)
    o_s, lse_s = oracle.forward(_bf16(q), _bf16(k + c), _bf16(v), 0.25)
    assert np.max(np.abs(o_s - o)) < 1e-13
    # the logsumexp shifts by scale * <q_i, c>
    shift = 0.25 * (q[0, 0] @ c).numpy()
    assert np.max(np.abs(lse_s[0] - lse[0] - shift)) < 1e-12


def test_row_and_head_selection_equals_full_result():
    x = make_inputs(2, 2, 64, 8, seed=12)
    o, lse = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=True, p_drop=0.2, seed=3)
    rows = [0, 5, 63]
    heads = [3, 1]
    os_, ls_ = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=True, p_drop=0.2, seed=3,
                              heads=heads, rows=rows)
    assert np.array_equal(os_, o[heads][:, rows])
    assert np.array_equal(ls_, lse[heads][:, rows])


def test_sample_rows_contains_ends():
    r = sample_rows(8192, 512, seed=2)
    assert r[0] == 0 and r[-1] == 8191 and len(r) == 512 and len(set(r)) == 512


# --------------------------------------------------------- backward pins

def _loss(q, k, v, dout, sc, causal, p_drop=0.0, seed=0):
    o, _ = oracle.forward(q, k, v, sc, causal=causal, p_drop=p_drop, seed=seed)
    return float(np.sum(o.reshape(dout.shape) * dout.numpy()))


@pytest.mark.parametrize("causal,p_drop", [(False, 0.0), (True, 0.0), (True, 0.3), (False, 0.3)])
def test_gradients_match_central_finite_differences(causal, p_drop):
    g = torch.Generator().manual_seed(21)
    B, H, N, d = 1, 2, 12, 6
    q, k, v, dout = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4))
    sc, seed = 0.45, 77
    dq, D, dev = oracle.backward_q(q, k, v, dout, sc, causal=causal, p_drop=p_drop, seed=seed)
    dk, dv = oracle.backward_kv(q, k, v, dout, sc, causal=causal, p_drop=p_drop, seed=seed)
    assert dev < 1e-12
    grads = {"q": dq.reshape(B, H, N, d), "k": dk.reshape(B, H, N, d), "v": dv.reshape(B, H, N, d)}
    h = 1e-6
    rng = np.random.default_rng(0)
    for name in ("q", "k", "v"):
        base = {"q": q, "k": k, "v": v}
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in (B, H, N, d))
            plus = {n: t.clone() for n, t in base.items()}
            minus = {n: t.clone() for n, t in base.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (_loss(plus["q"], plus["k"], plus["v"], dout, sc, causal, p_drop, seed)
                  - _loss(minus["q"], minus["k"], minus["v"], dout, sc, causal, p_drop, seed)) / (2 * h)
            an = grads[name][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd_fp64(causal):
    x = make_inputs(1, 2, 40, 16, seed=13)
    sc = 0.25
    q, k, v = (_f64(x[n]).requires_grad_(True) for n in ("q", "k", "v"))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=sc)
    o.backward(_f64(x["do"]))
    dq, D, dev = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], sc, causal=causal)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], sc, causal=causal)
    assert np.max(np.abs(dq - q.grad.reshape(2, 40, 16).numpy())) < 1e-11
    assert np.max(np.abs(dk - k.grad.reshape(2, 40, 16).numpy())) < 1e-11
    assert np.max(np.abs(dv - v.grad.reshape(2, 40, 16).numpy())) < 1e-11
    # D_i = <dO_i, O_i>
    ref_D = (o.detach() * _f64(x["do"])).sum(-1).reshape(2, 40).numpy()
    assert np.max(np.abs(D - ref_D)) < 1e-11


@pytest.mark.parametrize("causal,p_drop", [(False, 0.0), (True, 0.0), (True, 0.2)])
def test_backward_invariants(causal, p_drop):
    x = make_inputs(1, 2, 64, 8, seed=14)
    sc = 0.35
    dq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], sc, causal=causal, p_drop=p_drop, seed=5)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], sc, causal=causal, p_drop=p_drop, seed=5)
    # every row of dS sums to zero over its visible keys => sum_j dK_j = 0
    assert np.max(np.abs(dk.sum(axis=1))) < 1e-12
    if p_drop == 0.0:
        # sum_j dV_j = sum_i dO_i (rows of P sum to one)
        assert np.max(np.abs(dv.sum(axis=1) - _f64(x["do"]).reshape(2, 64, 8).sum(1).numpy())) < 1e-12
    if causal:
        # row 0 sees only key 0: dS_00 = P_00 (dP_00 - D_0) = 0
        assert np.max(np.abs(dq[:, 0])) < 1e-14


def test_key_selection_equals_full_result():
    x = make_inputs(1, 2, 48, 8, seed=15)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 0.3, causal=True, p_drop=0.1, seed=2)
    keys = [40, 7, 47]
    dks, dvs = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 0.3, causal=True, p_drop=0.1, seed=2,
                                  heads=[1], keys=keys)
    assert np.array_equal(dks[0], dk[1][keys])
    assert np.array_equal(dvs[0], dv[1][keys])


# ---------------------------------------------------------- dropout pins

def test_dropout_zero_probability_is_plain_attention():
    x = make_inputs(1, 2, 32, 8, seed=16)
    a = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=True)
    b = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=True, p_drop=0.0, seed=123)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_dropout_is_unbiased_and_leaves_lse_unchanged():
    """E_seed[O with dropout] = O without dropout (survivors scaled by 1/(1-p));
    the logsumexp is the undropped one for every seed."""
    x = make_inputs(1, 1, 16, 4, seed=17)
    sc, p = 0.5, 0.3
    o0, lse0 = oracle.forward(x["q"], x["k"], x["v"], sc)
    outs = []
    for s in range(3000):
        o, lse = oracle.forward(x["q"], x["k"], x["v"], sc, p_drop=p, seed=s)
        assert np.array_equal(lse, lse0)
        outs.append(o)
    outs = np.stack(outs)
    mean, std = outs.mean(0), outs.std(0) / math.sqrt(outs.shape[0])
    assert np.all(np.abs(mean - o0) < 5 * std + 1e-12)


def test_dropout_mask_is_what_the_forward_applies():
    """With one-hot V columns the output exposes P_ij Z_ij / (1-p) directly."""
    N = 16
    x = make_inputs(1, 1, N, 16, seed=18)
    eye = torch.eye(N, 16).reshape(1, 1, N, 16).to(torch.bfloat16)
    sc, p, seed = 0.4, 0.25, 99
    o, _ = oracle.forward(x["q"], x["k"], eye, sc, p_drop=p, seed=seed)
    o_plain, _ = oracle.forward(x["q"], x["k"], eye, sc)  # = P
    z = oracle.dropout_mask(1, 1, N, p, seed)[0]
    assert np.max(np.abs(o[0] - o_plain[0] * z / (1 - p))) < 1e-15


# ------------------------------------------------- pages' arithmetic pins

def test_pages_memory_arithmetic():
    from io_aware_exact_25_b200 import accounting
    ref = json.load(open(os.path.join(GOLDEN, "pages_memory_arithmetic.json")))
    a = ref["score_matrix_bytes_32k_16heads"]
    gib = accounting.score_matrix_bytes(a["B"], a["H"], a["N"], a["bytes_per_elem"]) / 2 ** 30
    assert abs(gib - a["expect_gib"]) < 1e-9
    b = ref["bandwidth_32k_1ms"]
    assert accounting.standard_attention_bandwidth(b["B"], b["N"], b["t_s"]) > b["expect_min_bytes_per_s"]
    c = ref["tile_saving_8192_512"]
    assert accounting.tiling_memory_saving(c["N"], c["tile"]) == c["expect_factor"]


# ----------------------------------------------------- block-sparse pins
# Block-sparse attention ("FlashAttention for Efficient Training", section
# 3.2, Block-Sparse Attention Support): a 0/1 mask over tile x tile blocks
# hides whole key blocks.  Small tiles keep these cases tiny.

def _random_block_mask(H, nt, seed, density=0.5, keep_diagonal=True):
    g = torch.Generator().manual_seed(seed)
    m = (torch.rand(H, nt, nt, generator=g) < density).to(torch.uint8)
    if keep_diagonal:
        m[:, torch.arange(nt), torch.arange(nt)] = 1
    return m


def _dense_mask(bm, N, tile, causal):
    """Element mask (True = visible) from a block mask, as torch SDPA takes it."""
    el = bm.to(torch.bool).repeat_interleave(tile, 1).repeat_interleave(tile, 2)[:, :N, :N]
    if causal:
        el = el & torch.ones(N, N, dtype=torch.bool).tril()
    return el


@pytest.mark.parametrize("causal,shared", [(False, False), (True, False), (False, True)])
def test_block_mask_matches_torch_element_mask(causal, shared):
    B, H, N, d, tile = 2, 3, 44, 8, 8           # 6 tiles, the last one ragged (4 rows)
    x = make_inputs(B, H, N, d, seed=31)
    nt = (N + tile - 1) // tile
    bm = _random_block_mask(1 if shared else H, nt, seed=32)
    sc = 0.3
    el = _dense_mask(bm, N, tile, causal).expand(H, N, N).unsqueeze(0)
    q, k, v = (_f64(x[n]).requires_grad_(True) for n in ("q", "k", "v"))
    o_ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=el, scale=sc)
    o_ref.backward(_f64(x["do"]))
    o, lse = oracle.forward(x["q"], x["k"], x["v"], sc, causal=causal, block_mask=bm, block=tile)
    assert np.max(np.abs(o - o_ref.detach().reshape(B * H, N, d).numpy())) < 1e-12
    s = (_f64(x["q"]) @ _f64(x["k"]).transpose(-1, -2)) * sc
    lse_ref = torch.logsumexp(s.masked_fill(~el, float("-inf")), dim=-1).reshape(B * H, N).numpy()
    assert np.max(np.abs(lse - lse_ref)) < 1e-12
    dq, _, dev = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], sc, causal=causal,
                                   block_mask=bm, block=tile)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], sc, causal=causal,
                                block_mask=bm, block=tile)
    assert dev < 1e-12
    for got, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        assert np.max(np.abs(got - ref.reshape(B * H, N, d).numpy())) < 1e-11


def test_all_ones_block_mask_is_dense_attention():
    x = make_inputs(1, 2, 40, 8, seed=33)
    ones = np.ones((1, 5, 5), np.uint8)
    for causal in (False, True):
        a = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=causal)
        b = oracle.forward(x["q"], x["k"], x["v"], 0.3, causal=causal, block_mask=ones, block=8)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
        ga = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 0.3, causal=causal)
        gb = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 0.3, causal=causal, block_mask=ones, block=8)
        assert np.array_equal(ga[0], gb[0]) and np.array_equal(ga[1], gb[1])


def test_block_diagonal_mask_is_independent_problems():
    """With only diagonal blocks, each tile is its own N = tile problem."""
    B, H, N, d, tile = 1, 2, 32, 8, 8
    x = make_inputs(B, H, N, d, seed=34)
    eye = np.eye(N // tile, dtype=np.uint8)[None]
    o, lse = oracle.forward(x["q"], x["k"], x["v"], 0.4, causal=True, block_mask=eye, block=tile)
    dq, _, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], 0.4, causal=True,
                                 block_mask=eye, block=tile)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], 0.4, causal=True,
                                block_mask=eye, block=tile)
    for a in range(N // tile):
        sl = slice(a * tile, (a + 1) * tile)
        sub = {n: x[n][:, :, sl].contiguous() for n in x}
        o_s, lse_s = oracle.forward(sub["q"], sub["k"], sub["v"], 0.4, causal=True)
        dq_s, _, _ = oracle.backward_q(sub["q"], sub["k"], sub["v"], sub["do"], 0.4, causal=True)
        dk_s, dv_s = oracle.backward_kv(sub["q"], sub["k"], sub["v"], sub["do"], 0.4, causal=True)
        assert np.max(np.abs(lse[:, sl] - lse_s)) < 1e-13
        for got, ref in ((o, o_s), (dq, dq_s), (dk, dk_s), (dv, dv_s)):
            assert np.max(np.abs(got[:, sl] - ref)) < 1e-13


def test_rows_that_see_no_key():
    """A query tile whose mask row is all zero: O = 0, lse = -inf, dQ = 0, and
    its rows add nothing to dK and dV (the other rows match torch run on them
    alone)."""
    B, H, N, d, tile = 1, 2, 40, 8, 8
    x = make_inputs(B, H, N, d, seed=35)
    bm = np.ones((H, 5, 5), np.uint8)
    bm[0, 2, :] = 0                               # head 0: rows 16..23 see nothing
    bm[1, 4, :] = 0                               # head 1: the last tile
    sc = 0.3
    o, lse = oracle.forward(x["q"], x["k"], x["v"], sc, block_mask=bm, block=tile)
    dq, D, _ = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], sc, block_mask=bm, block=tile)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], sc, block_mask=bm, block=tile)
    empty = {0: slice(16, 24), 1: slice(32, 40)}
    for h, sl in empty.items():
        assert np.all(o[h, sl] == 0.0) and np.all(np.isneginf(lse[h, sl]))
        assert np.all(dq[h, sl] == 0.0) and np.all(D[h, sl] == 0.0)
        keep = [i for i in range(N) if not (sl.start <= i < sl.stop)]
        q = _f64(x["q"][0, h, keep]).requires_grad_(True)
        k = _f64(x["k"][0, h]).requires_grad_(True)
        v = _f64(x["v"][0, h]).requires_grad_(True)
        o_ref = torch.softmax((q @ k.T) * sc, dim=-1) @ v
        o_ref.backward(_f64(x["do"][0, h, keep]))
        assert np.max(np.abs(o[h, keep] - o_ref.detach().numpy())) < 1e-12
        assert np.max(np.abs(dk[h] - k.grad.numpy())) < 1e-11
        assert np.max(np.abs(dv[h] - v.grad.numpy())) < 1e-11


def test_block_mask_shape_is_checked():
    x = make_inputs(1, 2, 40, 8, seed=36)
    with pytest.raises(ValueError):
        oracle.forward(x["q"], x["k"], x["v"], 0.3, block_mask=np.ones((1, 4, 4), np.uint8), block=8)
    with pytest.raises(ValueError):
        oracle.forward(x["q"], x["k"], x["v"], 0.3, block_mask=np.ones((3, 5, 5), np.uint8), block=8)


# ------------------------------------------------- variable sequence lengths
#
# "FlashAttention for Efficient Training", section 5.2 (Efficient Padding and
# Masking): a score is -inf unless its key lies within the sequence.  With a
# length L_b per batch entry, rows and keys at or beyond L_b are padding.

def _varlen_all(x, sc, causal, lens, p=0.0, seed=0):
    kw = dict(causal=causal, p_drop=p, seed=seed, seqlens=lens)
    o, lse = oracle.forward(x["q"], x["k"], x["v"], sc, **kw)
    dq, D, dev = oracle.backward_q(x["q"], x["k"], x["v"], x["do"], sc, **kw)
    dk, dv = oracle.backward_kv(x["q"], x["k"], x["v"], x["do"], sc, **kw)
    assert dev < 1e-12
    return o, lse, dq, D, dk, dv


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_rows_equal_torch_on_each_unpadded_sequence(causal):
    """Each batch entry's real rows equal torch fp64 SDPA + autograd run on
    that sequence alone; padding rows are exactly O = 0, lse = -inf, dQ = 0
    and padding keys exactly dK = dV = 0."""
    B, H, N, d = 4, 2, 24, 8
    lens = [24, 13, 1, 0]
    x = make_inputs(B, H, N, d, seed=41)
    sc = 0.35
    o, lse, dq, D, dk, dv = _varlen_all(x, sc, causal, lens)
    shape = (B, H, N, d)
    o, dq, dk, dv = (t.reshape(shape) for t in (o, dq, dk, dv))
    lse, D = lse.reshape(B, H, N), D.reshape(B, H, N)
    for b, L in enumerate(lens):
        pad = slice(L, N)
        assert np.all(o[b, :, pad] == 0.0) and np.all(np.isneginf(lse[b, :, pad]))
        assert np.all(dq[b, :, pad] == 0.0) and np.all(D[b, :, pad] == 0.0)
        assert np.all(dk[b, :, pad] == 0.0) and np.all(dv[b, :, pad] == 0.0)
        if L == 0:
            continue
        q, k, v = (_f64(x[n][b:b + 1, :, :L]).requires_grad_(True) for n in ("q", "k", "v"))
        o_ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=sc)
        o_ref.backward(_f64(x["do"][b:b + 1, :, :L]))
        s = (q.detach() @ k.detach().transpose(-1, -2)) * sc
        if causal:
            s = s.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), float("-inf"))
        lse_ref = torch.logsumexp(s, dim=-1)[0].numpy()
        assert np.max(np.abs(o[b, :, :L] - o_ref.detach()[0].numpy())) < 1e-12
        assert np.max(np.abs(lse[b, :, :L] - lse_ref)) < 1e-12
        for got, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
            assert np.max(np.abs(got[b, :, :L] - ref[0].numpy())) < 1e-11


def test_varlen_padding_values_never_enter_a_result():
    """Rewriting every padding row of Q, K, V and dO changes no bit of any
    output."""
    B, H, N, d = 3, 2, 20, 8
    lens = [20, 7, 12]
    x = make_inputs(B, H, N, d, seed=42)
    y = {n: t.clone() for n, t in x.items()}
    g = torch.Generator().manual_seed(43)
    for b, L in enumerate(lens):
        for n in y:
            y[n][b, :, L:] = (torch.randn(H, N - L, d, generator=g) * 50).to(torch.bfloat16)
    for causal in (False, True):
        a = _varlen_all(x, 0.3, causal, lens, p=0.2, seed=9)
        c = _varlen_all(y, 0.3, causal, lens, p=0.2, seed=9)
        for u, w in zip(a, c):
            assert np.array_equal(u, w)


def test_varlen_with_equal_lengths_is_the_shorter_problem_with_dropout():
    """All lengths L < N: the padded problem equals the unpadded N = L batch
    bit for bit, dropout included (the mask is indexed by the batch entry and
    the positions within the sequence)."""
    B, H, N, d, L = 2, 2, 32, 8, 19
    x = make_inputs(B, H, N, d, seed=44)
    sub = {n: t[:, :, :L].contiguous() for n, t in x.items()}
    for causal in (False, True):
        a = _varlen_all(x, 0.4, causal, [L] * B, p=0.25, seed=11)
        c = _varlen_all(sub, 0.4, causal, None, p=0.25, seed=11)
        BH = B * H
        for u, w in zip(a, c):
            u = u.reshape(BH, N, -1) if u.ndim == 3 else u.reshape(BH, N, 1)
            w = w.reshape(BH, L, -1) if w.ndim == 3 else w.reshape(BH, L, 1)
            assert np.array_equal(u[:, :L], w)


def test_varlen_lengths_are_checked():
    x = make_inputs(2, 1, 8, 8, seed=45)
    for bad in ([8], [9, 1], [-1, 3]):
        with pytest.raises(ValueError):
            oracle.forward(x["q"], x["k"], x["v"], 0.3, seqlens=bad)
