"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export every symbol ``include/fa.h`` declares, and
reject invalid arguments with the documented status codes before touching
the device.
"""
import ctypes
import os
import re

import pytest

from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "fa_fwd" in names and "fa_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(binding.EXPORTS) == set(names)


def test_bounds_checking_build_exports_the_same_symbols(lib):
    """libfa_sm100_debug.so (FA_DEBUG) is the same ABI with its checks on;
    only it answers the record query (no device is touched for either)."""
    dbg = ctypes.CDLL(binding.DEBUG_LIB_PATH)
    for n in declared_functions():
        assert hasattr(dbg, n), n
    assert lib.fa_debug_build() == 0 and dbg.fa_debug_build() == 1
    out = (ctypes.c_longlong * 6)()
    assert lib.fa_debug_bounds_record(out, None) == binding.FA_ERR_UNSUPPORTED
    assert dbg.fa_debug_bounds_record(None, None) == binding.FA_ERR_INVALID_ARG


def test_status_codes_match_header(lib):
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    codes = dict((k, int(v)) for k, v in re.findall(r"(FA_[A-Z_]+)\s*=\s*(-?\d+)", text))
    for k, v in codes.items():
        assert getattr(binding, k) == v
        assert lib.fa_strerror(v) and lib.fa_strerror(v).decode() != "unknown status"
    assert lib.fa_strerror(12345).decode() == "unknown status"
    assert lib.fa_version() == 200


def _fwd(lib, q=16, k=16, v=16, o=16, lse=16, B=1, H=1, N=128, d=64, scale=0.125, causal=0, p=0.0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, p, 0, None)


def _bwd(lib, ptr=16, lse=16, B=1, H=1, N=128, d=64, scale=0.125, causal=0, p=0.0, ws=16, wsb=1 << 30):
    return lib.fa_bwd(ptr, ptr, ptr, ptr, ptr, lse, ptr, ptr, ptr, B, H, N, d, scale, causal, p, 0, ws, wsb,
                      None)


def test_invalid_arguments_are_rejected_before_launch(lib):
    assert _fwd(lib, d=96) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, d=256) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, B=-1) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, N=-5) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf")) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, causal=2) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, p=1.0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, p=-0.1) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, q=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, lse=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, q=24) == binding.FA_ERR_ALIGNMENT      # 8-byte aligned only
    assert _fwd(lib, o=18) == binding.FA_ERR_ALIGNMENT
    assert _fwd(lib, lse=18) == binding.FA_ERR_ALIGNMENT
    assert _fwd(lib, B=1 << 25) == binding.FA_ERR_TOO_LARGE
    assert _bwd(lib, ws=None) == binding.FA_ERR_WORKSPACE
    assert _bwd(lib, wsb=100) == binding.FA_ERR_WORKSPACE
    assert _bwd(lib, ws=24) == binding.FA_ERR_ALIGNMENT
    assert _bwd(lib, ptr=None) == binding.FA_ERR_INVALID_ARG
    assert _bwd(lib, d=80) == binding.FA_ERR_UNSUPPORTED
    assert _bwd(lib, p=1.5) == binding.FA_ERR_INVALID_ARG


def test_strided_entry_points_check_strides(lib):
    S = binding.FaStrides
    good = (S * 8)(*[S(3 * 128 * 64, 128 * 64, 64)] * 8)
    bad = (S * 8)(*[S(3 * 128 * 64, 128 * 64, 63)] * 8)  # 126-byte rows: misaligned
    args = (1, 3, 128, 64, 0.125, 0, 0.0, 0)
    assert lib.fa_fwd_strided(16, 16, 16, 16, 16, bad, *args, None) == binding.FA_ERR_ALIGNMENT
    assert lib.fa_fwd_strided(16, 16, 16, 16, 16, None, *args, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_strided(16, 16, 16, 16, 16, 16, 16, 16, 16, bad, *args, 16, 1 << 30, None) \
        == binding.FA_ERR_ALIGNMENT
    assert lib.fa_bwd_strided(16, 16, 16, 16, 16, 16, 16, 16, 16, good, *args, None, 0, None) \
        == binding.FA_ERR_WORKSPACE


def test_splitkv_workspace_and_arguments(lib):
    B, H, N, d = 1, 2, 1000, 128
    rows = B * H * N * 3

    def up(x):
        return (x + 255) // 256 * 256
    assert lib.fa_fwd_splitkv_workspace_size(B, H, N, d, 3) == up(rows * d * 4) + up(rows * 4)
    assert lib.fa_fwd_splitkv_workspace_size(B, H, N, d, 1) == 0
    assert lib.fa_fwd_splitkv_workspace_size(B, H, N, d, 65) == 0
    args = (B, H, N, d, 0.1, 0, 0.0, 0)
    assert lib.fa_fwd_splitkv(16, 16, 16, 16, 16, *args, 0, 16, 1 << 30, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_splitkv(16, 16, 16, 16, 16, *args, 3, None, 0, None) == binding.FA_ERR_WORKSPACE
    assert lib.fa_fwd_splitkv(16, 16, 16, 16, 16, *args, 3, 16, 100, None) == binding.FA_ERR_WORKSPACE
    assert lib.fa_splitkv_suggest(2, 16, 8192, 128) == 1       # 512 CTAs fill the GPU
    assert lib.fa_splitkv_suggest(1, 2, 16384, 128) == 1       # 128 CTAs: more than half full
    assert lib.fa_splitkv_suggest(1, 1, 16384, 128) == 2       # 64 CTAs -> one wave of 128


def test_blocksparse_arguments(lib):
    args = (1, 3, 300, 64, 0.125, 0, 0.0, 0)
    # null mask, or a mask shared by neither one head nor all H heads
    assert lib.fa_fwd_blocksparse(16, 16, 16, 16, 16, None, *args, None, 1, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_blocksparse(16, 16, 16, 16, 16, None, *args, 16, 2, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_blocksparse(16, 16, 16, 16, 16, 16, 16, 16, 16, None, *args, 16, 0, 16, 1 << 30, None) \
        == binding.FA_ERR_INVALID_ARG
    # more than 4096 key tiles
    big = (1, 1, 4096 * 128 + 1, 64, 0.125, 0, 0.0, 0)
    assert lib.fa_fwd_blocksparse(16, 16, 16, 16, 16, None, *big, 16, 1, None) == binding.FA_ERR_TOO_LARGE
    assert lib.fa_bwd_blocksparse(16, 16, 16, 16, 16, 16, 16, 16, 16, None, *big, 16, 1, 16, 1 << 40, None) \
        == binding.FA_ERR_TOO_LARGE
    # workspace still checked; empty problems are no-ops
    assert lib.fa_bwd_blocksparse(16, 16, 16, 16, 16, 16, 16, 16, 16, None, *args, 16, 3, None, 0, None) \
        == binding.FA_ERR_WORKSPACE
    assert lib.fa_fwd_blocksparse(None, None, None, None, None, None, 1, 1, 0, 64, 0.1, 0, 0.0, 0, None, 1,
                                  None) == binding.FA_OK


def test_empty_problems_are_noops(lib):
    # nothing to do: success without touching the (absent) device or pointers
    assert _fwd(lib, q=None, k=None, v=None, o=None, lse=None, N=0) == binding.FA_OK
    assert _fwd(lib, q=None, k=None, v=None, o=None, lse=None, B=0) == binding.FA_OK
    assert _bwd(lib, ptr=None, lse=None, H=0, ws=None, wsb=0) == binding.FA_OK
    assert lib.fa_dropout_mask(1, 1, 0, 0.1, 0, None, 0, None, 0, None, None) == binding.FA_OK
    assert lib.fa_debug_exp2_poly(None, None, 0, None) == binding.FA_OK


def test_exp2_hook_rejects_bad_arguments(lib):
    assert lib.fa_debug_exp2_poly(None, None, -1, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_debug_exp2_poly(None, None, 4, None) == binding.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 128, 64), (2, 16, 8192, 128), (1, 3, 300, 128), (1, 1, 1, 64)])
def test_workspace_size_formula(lib, B, H, N, d):
    npad = (N + 127) // 128 * 128

    def up(x):
        return (x + 255) // 256 * 256
    # fp32 dQ accumulator, scaled lse and D rows, the backward's item counter
    expect = up(B * H * npad * d * 4) + 2 * up(B * H * npad * 4) + 256
    assert lib.fa_bwd_workspace_size(B, H, N, d) == expect
    assert lib.fa_bwd_dq_accumulator_bytes(B, H, N, d) == up(B * H * npad * d * 4)
    assert lib.fa_bwd_workspace_size(B, H, N, 96) == 0
    assert lib.fa_bwd_workspace_size(0, H, N, d) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.fwd(x, x, x)


def test_varlen_arguments_are_rejected_before_launch(lib):
    S = (binding.FaStrides * 8)(*[binding.FaStrides(0, 64, 64 * 4)] * 8)

    def fwd(cu=16, used=None, B=2, H=4, maxs=128, T=300, d=64, strides=S, q=16):
        return lib.fa_fwd_varlen(q, 16, 16, 16, 16, strides, cu, used, B, H, maxs, T, d, 0.125, 0, 0.0, 0, None)

    def bwd(cu=16, ws=16, wsb=1 << 30, d=64):
        return lib.fa_bwd_varlen(16, 16, 16, 16, 16, 16, 16, 16, 16, S, cu, None, 2, 4, 128, 300, d, 0.125, 0, 0.0,
                                 0, ws, wsb, None)

    assert fwd(cu=None) == binding.FA_ERR_INVALID_ARG
    assert fwd(cu=18) == binding.FA_ERR_ALIGNMENT
    assert fwd(used=18) == binding.FA_ERR_ALIGNMENT
    assert fwd(q=24) == binding.FA_ERR_ALIGNMENT
    assert fwd(d=96) == binding.FA_ERR_UNSUPPORTED
    assert fwd(T=-1) == binding.FA_ERR_INVALID_ARG
    assert fwd(strides=None) == binding.FA_ERR_INVALID_ARG
    bad = (binding.FaStrides * 4)(*[binding.FaStrides(0, 64, 60)] * 4)   # token stride of 120 bytes
    assert fwd(strides=bad) == binding.FA_ERR_ALIGNMENT
    # empty problems launch nothing (no pointer is inspected)
    assert fwd(cu=None, T=0) == binding.FA_OK
    assert fwd(cu=None, B=0) == binding.FA_OK
    assert bwd(ws=None) == binding.FA_ERR_WORKSPACE
    assert bwd(wsb=100) == binding.FA_ERR_WORKSPACE
    assert bwd(cu=None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_varlen_workspace_size(2, 4, 128, 64) == lib.fa_bwd_workspace_size(2, 4, 128, 64)


def test_key_window_arguments_are_rejected_before_launch(lib):
    def part(kb, ke, N=1000, d=64, k=16):
        return lib.fa_fwd_partial(16, k, 16, 16, 16, 1, 2, N, d, 0.125, 1, 0.0, 0, kb, ke, None)

    def rng(kb, ke, N=1000):
        return lib.fa_bwd_recompute_range(16, 16, 16, 16, 16, 16, 1, 2, N, 64, 0.125, 1, 0.0, 0, kb, ke, 16,
                                          1 << 30, None)

    for kb, ke in ((100, 1000), (0, 1001), (256, 200), (-128, 256), (0, 300)):
        assert part(kb, ke) == binding.FA_ERR_INVALID_ARG, (kb, ke)
        assert rng(kb, ke) == binding.FA_ERR_INVALID_ARG, (kb, ke)
    assert part(0, 256, d=80) == binding.FA_ERR_UNSUPPORTED
    assert part(0, 256, k=24) == binding.FA_ERR_ALIGNMENT
    assert rng(256, 256) == binding.FA_OK  # an empty window adds nothing and launches nothing
    assert lib.fa_merge_partials(16, 16, 0, 16, 16, 1, 2, 100, 64, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_merge_partials(16, 18, 2, 16, 16, 1, 2, 100, 64, None) == binding.FA_ERR_ALIGNMENT


def test_weight_partial_arguments_are_rejected_before_launch(lib):
    def w(po=16, al=16, S=2, part=0, lse=16, d=64, B=1):
        return lib.fa_weight_partial(po, al, S, part, lse, B, 2, 100, d, None)

    for S, part in ((0, 0), (2, 2), (2, -1), (4097, 0)):
        assert w(S=S, part=part) == binding.FA_ERR_INVALID_ARG, (S, part)
    assert w(d=80) == binding.FA_ERR_UNSUPPORTED
    assert w(po=None) == binding.FA_ERR_INVALID_ARG and w(al=None) == binding.FA_ERR_INVALID_ARG
    assert w(po=24) == binding.FA_ERR_ALIGNMENT and w(al=18) == binding.FA_ERR_ALIGNMENT
    assert w(lse=18) == binding.FA_ERR_ALIGNMENT
    assert w(B=0) == binding.FA_OK and w(B=-1) == binding.FA_ERR_INVALID_ARG  # empty: nothing launched
    # B*H*N*num_parts = 2^30 * 2 * 100 * 4096 > 2^40 is refused before any launch
    assert lib.fa_weight_partial(16, 16, 4096, 0, 16, 1 << 30, 2, 100, 64, None) == binding.FA_ERR_TOO_LARGE
