"""Thin ctypes binding over the C ABI in ``include/fa.h``.

Argument marshalling only: every step of the attention path runs in the CUDA
kernels of ``libfa_sm100.so``.  Tensors are torch CUDA tensors (torch supplies
device memory and the current stream); outputs are allocated here with torch
when the caller does not pass them.  There is no CPU fallback: a missing
library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_sm100.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libfa_sm100_debug.so")  # the bounds-checking build (FA_DEBUG)

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_ALIGNMENT = -3
FA_ERR_WORKSPACE = -4
FA_ERR_CUDA = -5
FA_ERR_DEVICE = -6
FA_ERR_TOO_LARGE = -7

EXPORTS = ("fa_fwd", "fa_fwd_strided", "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_size",
           "fa_splitkv_suggest", "fa_bwd", "fa_bwd_strided", "fa_bwd_workspace_size", "fa_bwd_prepare", "fa_bwd_recompute",
           "fa_bwd_finalize", "fa_bwd_noalloc", "fa_fwd_blocksparse", "fa_bwd_blocksparse",
           "fa_bwd_recompute_blocksparse", "fa_debug_fwd_timeout", "fa_debug_exp2_poly",
           "fa_debug_build", "fa_debug_bounds_record",
           "fa_fwd_varlen", "fa_bwd_varlen", "fa_bwd_varlen_workspace_size",
           "fa_fwd_partial", "fa_merge_partials", "fa_weight_partial", "fa_bwd_dq_accumulator_bytes", "fa_bwd_recompute_range",
           "fa_dropout_mask", "fa_strerror",
           "fa_last_cuda_error", "fa_get_device_error", "fa_version")

NOALLOC_SCRATCH_BYTES = 32 << 20

_lock = threading.Lock()
_lib = None


class FaStrides(ctypes.Structure):
    """Element strides (batch, head, row) of a [B,H,N,d] tensor, d contiguous."""
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("n", ctypes.c_int64)]


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} ({status})")


def load() -> ctypes.CDLL:
    """Load ``libfa_sm100.so`` (raises if it has not been built); every
    function of this module calls through it.  With ``FA_BOUNDS_CHECK=1`` in
    the environment the bounds-checking build is loaded instead."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        _lib = _open(DEBUG_LIB_PATH if os.environ.get("FA_BOUNDS_CHECK") == "1" else LIB_PATH)
        return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Route every call of this module through another build of the library
    (``DEBUG_LIB_PATH``, the bounds-checking build) inside the block."""
    global _lib
    lib = _open(path)
    with _lock:
        saved = _lib
        _lib = lib
    try:
        yield lib
    finally:
        with _lock:
            _lib = saved


def debug_bounds_record(stream=None) -> list:
    """The bounds-checking build's record of its first failed check
    ({failed checks, site, offset, limit, block, thread}), cleared by reading."""
    out = (ctypes.c_longlong * 6)()
    _call(load().fa_debug_bounds_record(out, _stream(stream)), "fa_debug_bounds_record")
    return list(out)


def _open(path: str) -> ctypes.CDLL:
    """Open one build of the library and declare its signatures."""
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing; build it with io_aware_exact_25_b200.build.build()")
    lib = ctypes.CDLL(path)
    vp, I, F, U64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, vp]
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, I, vp, SZ, vp]
    lib.fa_fwd_splitkv_workspace_size.argtypes = [I, I, I, I, I]
    lib.fa_fwd_splitkv_workspace_size.restype = SZ
    lib.fa_splitkv_suggest.argtypes = [I, I, I, I]
    lib.fa_splitkv_suggest.restype = I
    SP = ctypes.POINTER(FaStrides)
    lib.fa_fwd_strided.argtypes = [vp, vp, vp, vp, vp, SP, I, I, I, I, F, I, F, U64, vp]
    lib.fa_bwd_strided.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, SP, I, I, I, I, F, I, F, U64, vp, SZ,
                                   vp]
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, vp, SZ, vp]
    lib.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, SP, I, I, I, I, F, I, F, U64, vp, I, vp]
    lib.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, SP, I, I, I, I, F, I, F, U64, vp, I,
                                       vp, SZ, vp]
    lib.fa_bwd_recompute_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, vp, I, vp, SZ,
                                                 vp]
    lib.fa_debug_fwd_timeout.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, vp]
    lib.fa_debug_exp2_poly.argtypes = [vp, vp, I, vp]
    lib.fa_debug_bounds_record.argtypes = [vp, vp]
    lib.fa_bwd_workspace_size.argtypes = [I, I, I, I]
    lib.fa_bwd_workspace_size.restype = SZ
    lib.fa_bwd_prepare.argtypes = [vp, vp, vp, I, I, I, I, vp, SZ, vp]
    lib.fa_bwd_recompute.argtypes = [vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, vp, SZ, vp]
    lib.fa_bwd_finalize.argtypes = [vp, I, I, I, I, F, vp, SZ, vp]
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, vp]
    lib.fa_dropout_mask.argtypes = [I, I, I, F, U64, vp, I, vp, I, vp, vp]
    lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, SP, vp, vp, I, I, I, I, I, F, I, F, U64, vp]
    lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, SP, vp, vp, I, I, I, I, I, F, I, F, U64,
                                  vp, SZ, vp]
    lib.fa_bwd_varlen_workspace_size.argtypes = [I, I, I, I]
    lib.fa_bwd_varlen_workspace_size.restype = SZ
    lib.fa_fwd_partial.argtypes = [vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, I, I, vp]
    lib.fa_merge_partials.argtypes = [vp, vp, I, vp, vp, I, I, I, I, vp]
    lib.fa_weight_partial.argtypes = [vp, vp, I, I, vp, I, I, I, I, vp]
    lib.fa_bwd_dq_accumulator_bytes.argtypes = [I, I, I, I]
    lib.fa_bwd_dq_accumulator_bytes.restype = SZ
    lib.fa_bwd_recompute_range.argtypes = [vp, vp, vp, vp, vp, vp, I, I, I, I, F, I, F, U64, I, I, vp, SZ, vp]
    lib.fa_strerror.argtypes = [I]
    lib.fa_strerror.restype = ctypes.c_char_p
    lib.fa_get_device_error.argtypes = [vp]
    for fn in (lib.fa_fwd, lib.fa_fwd_splitkv, lib.fa_fwd_strided, lib.fa_bwd_strided, lib.fa_bwd,
               lib.fa_bwd_prepare, lib.fa_bwd_recompute, lib.fa_bwd_finalize, lib.fa_bwd_noalloc,
               lib.fa_fwd_blocksparse, lib.fa_bwd_blocksparse, lib.fa_bwd_recompute_blocksparse,
               lib.fa_debug_fwd_timeout, lib.fa_debug_exp2_poly, lib.fa_fwd_varlen, lib.fa_bwd_varlen, lib.fa_fwd_partial,
               lib.fa_merge_partials, lib.fa_weight_partial, lib.fa_bwd_recompute_range,
               lib.fa_dropout_mask, lib.fa_get_device_error,
               lib.fa_last_cuda_error, lib.fa_version, lib.fa_debug_build, lib.fa_debug_bounds_record):
        fn.restype = I
    return lib


def strerror(status: int) -> str:
    return load().fa_strerror(int(status)).decode()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _check_inputs(*ts):
    """[B,H,N,d] bf16 CUDA tensors (any strides with a contiguous last dim)."""
    shape = ts[0].shape
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (there is no CPU path)")
        if t.dtype != torch.bfloat16:
            raise ValueError("q, k, v, o, dO must be bf16")
        if t.dim() != 4 or t.shape != shape:
            raise ValueError("tensors must be [B,H,N,d] of one shape")
        if t.stride(-1) != 1:
            raise ValueError("the head dimension must be contiguous")


def _check_dense(*ts):
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("this entry point takes dense [B,H,N,d] tensors")


def _strides(*ts):
    arr = (FaStrides * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = FaStrides(t.stride(0), t.stride(1), t.stride(2))
    return arr


def _check_block_mask(m, q):
    """Block mask: uint8 CUDA tensor [1 or H, nt, nt], nt = ceil(N / 128), dense."""
    B, H, N, d = q.shape
    nt = (N + 127) // 128
    if not m.is_cuda or m.device != q.device:
        raise ValueError("block_mask must be a CUDA tensor on the inputs' device")
    if m.dtype not in (torch.uint8, torch.bool):
        raise ValueError("block_mask must be uint8 or bool")
    if m.dim() != 3 or m.shape[0] not in (1, H) or tuple(m.shape[1:]) != (nt, nt):
        raise ValueError(f"block_mask must be [1 or {H}, {nt}, {nt}], got {tuple(m.shape)}")
    if not m.is_contiguous():
        raise ValueError("block_mask must be contiguous")
    return m.view(torch.uint8) if m.dtype == torch.bool else m


def _call(rc: int, what: str):
    if rc != FA_OK:
        raise FaError(rc, what)


def fwd(q, k, v, causal=False, scale=None, dropout_p=0.0, seed=0, o=None, lse=None, stream=None,
        block_mask=None):
    """O and lse of exact attention via ``fa_fwd_strided``, or
    ``fa_fwd_blocksparse`` when a ``block_mask`` ([1 or H, nt, nt] uint8 over
    128 x 128 blocks) is given."""
    _check_inputs(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_inputs(q, o)
    if block_mask is not None:
        m = _check_block_mask(block_mask, q)
        rc = load().fa_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _strides(q, k, v, o), B, H,
                                       N, d, float(scale), int(bool(causal)), float(dropout_p), int(seed), _ptr(m),
                                       int(m.shape[0]), _stream(stream))
        _call(rc, "fa_fwd_blocksparse")
        return o, lse
    rc = load().fa_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _strides(q, k, v, o), B, H, N, d,
                               float(scale), int(bool(causal)), float(dropout_p), int(seed), _stream(stream))
    _call(rc, "fa_fwd")
    return o, lse


def fwd_splitkv(q, k, v, causal=False, scale=None, dropout_p=0.0, seed=0, num_splits=None, o=None, lse=None,
                workspace=None, stream=None):
    """O and lse via ``fa_fwd_splitkv`` (dense [B,H,N,d] tensors).  The split
    count defaults to ``fa_splitkv_suggest``."""
    _check_inputs(q, k, v)
    _check_dense(q, k, v)
    B, H, N, d = q.shape
    lib = load()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits is None:
        num_splits = int(lib.fa_splitkv_suggest(B, H, N, d))
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    need = int(lib.fa_fwd_splitkv_workspace_size(B, H, N, d, int(num_splits)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = lib.fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                            int(bool(causal)), float(dropout_p), int(seed), int(num_splits), _ptr(workspace),
                            int(workspace.numel() * workspace.element_size()), _stream(stream))
    _call(rc, "fa_fwd_splitkv")
    return o, lse


def bwd_workspace_size(B, H, N, d) -> int:
    return int(load().fa_bwd_workspace_size(B, H, N, d))


def bwd(q, k, v, o, dout, lse, causal=False, scale=None, dropout_p=0.0, seed=0, dq=None, dk=None,
        dv=None, workspace=None, stream=None, block_mask=None):
    """dQ, dK, dV via ``fa_bwd_strided`` (or ``fa_bwd_blocksparse`` with the
    forward's ``block_mask``); allocates the workspace with torch if not given."""
    _check_inputs(q, k, v, o, dout)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_inputs(q, dq, dk, dv)
    if block_mask is not None:
        m = _check_block_mask(block_mask, q)
        rc = load().fa_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                       _ptr(dk), _ptr(dv), _strides(q, k, v, o, dout, dq, dk, dv), B, H, N, d,
                                       float(scale), int(bool(causal)), float(dropout_p), int(seed), _ptr(m),
                                       int(m.shape[0]), _ptr(workspace),
                                       int(workspace.numel() * workspace.element_size()), _stream(stream))
        _call(rc, "fa_bwd_blocksparse")
        return dq, dk, dv
    rc = load().fa_bwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                               _ptr(dv), _strides(q, k, v, o, dout, dq, dk, dv), B, H, N, d, float(scale),
                               int(bool(causal)), float(dropout_p), int(seed), _ptr(workspace),
                               int(workspace.numel() * workspace.element_size()), _stream(stream))
    _call(rc, "fa_bwd")
    return dq, dk, dv


def bwd_stages(q, k, v, o, dout, lse, causal=False, scale=None, dropout_p=0.0, seed=0, dq=None,
               dk=None, dv=None, workspace=None, stream=None):
    """The backward as its three C-ABI stages (prepare, recompute, finalize);
    dense [B,H,N,d] tensors only."""
    _check_inputs(q, k, v, o, dout)
    _check_dense(q, k, v, o, dout)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    wsb = int(workspace.numel() * workspace.element_size())
    s = _stream(stream)
    lib = load()
    _call(lib.fa_bwd_prepare(_ptr(o), _ptr(dout), _ptr(lse), B, H, N, d, _ptr(workspace), wsb, s),
          "fa_bwd_prepare")
    _call(lib.fa_bwd_recompute(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk), _ptr(dv), B, H, N, d,
                               float(scale), int(bool(causal)), float(dropout_p), int(seed),
                               _ptr(workspace), wsb, s), "fa_bwd_recompute")
    _call(lib.fa_bwd_finalize(_ptr(dq), B, H, N, d, float(scale), _ptr(workspace), wsb, s),
          "fa_bwd_finalize")
    return dq, dk, dv


def bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, causal=False, scale=None, dropout_p=0.0, seed=0,
                stream=None):
    """dQ, dK, dV via ``fa_bwd_noalloc`` into caller-provided outputs.

    Uses the library's static scratch instead of a workspace, so nothing is
    allocated here either (the outputs must be passed in).
    """
    _check_inputs(q, k, v, o, dout, dq, dk, dv)
    _check_dense(q, k, v, o, dout, dq, dk, dv)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = load().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, H, N, d, float(scale), int(bool(causal)), float(dropout_p),
                               int(seed), _stream(stream))
    _call(rc, "fa_bwd_noalloc")
    return dq, dk, dv


def _check_varlen(ts, cu_seqlens, seqused):
    """Token-major [T, H, d] bf16 CUDA tensors of one shape (d contiguous),
    int32 CUDA offsets [B + 1] and optional int32 lengths [B]."""
    shape = ts[0].shape
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (there is no CPU path)")
        if t.dtype != torch.bfloat16:
            raise ValueError("q, k, v, o, dO must be bf16")
        if t.dim() != 3 or t.shape != shape:
            raise ValueError("variable-length tensors must be [total_tokens, H, d] of one shape")
        if t.stride(-1) != 1:
            raise ValueError("the head dimension must be contiguous")
    for name, a, n in (("cu_seqlens", cu_seqlens, None), ("seqused", seqused, None)):
        if a is None:
            continue
        if not a.is_cuda or a.dtype != torch.int32 or a.dim() != 1 or not a.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA vector")
    B = cu_seqlens.numel() - 1
    if B < 0:
        raise ValueError("cu_seqlens needs B + 1 >= 1 entries")
    if seqused is not None and seqused.numel() != B:
        raise ValueError("seqused must have B entries")
    return B


def _tok_strides(*ts):
    arr = (FaStrides * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = FaStrides(0, t.stride(1), t.stride(0))
    return arr


def fwd_varlen(q, k, v, cu_seqlens, max_seqlen, seqused=None, causal=False, scale=None, dropout_p=0.0, seed=0,
               o=None, lse=None, stream=None):
    """O [T, H, d] and lse [H, T] of a variable-length batch via
    ``fa_fwd_varlen``: sequence b is tokens ``cu_seqlens[b]`` to
    ``cu_seqlens[b+1]`` of the token-major tensors (its first ``seqused[b]``
    tokens if given); ``max_seqlen`` bounds the slot sizes."""
    B = _check_varlen((q, k, v), cu_seqlens, seqused)
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    _check_varlen((q, o), cu_seqlens, seqused)
    rc = load().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _tok_strides(q, k, v, o),
                              _ptr(cu_seqlens), _ptr(seqused), B, H, int(max_seqlen), T, d, float(scale),
                              int(bool(causal)), float(dropout_p), int(seed), _stream(stream))
    _call(rc, "fa_fwd_varlen")
    return o, lse


def bwd_varlen(q, k, v, o, dout, lse, cu_seqlens, max_seqlen, seqused=None, causal=False, scale=None,
               dropout_p=0.0, seed=0, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV [T, H, d] of a variable-length batch via ``fa_bwd_varlen``
    (the forward's ``lse`` [H, T]); allocates the workspace with torch if not
    given."""
    B = _check_varlen((q, k, v, o, dout), cu_seqlens, seqused)
    T, H, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check_varlen((q, dq, dk, dv), cu_seqlens, seqused)
    lib = load()
    need = int(lib.fa_bwd_varlen_workspace_size(B, H, int(max_seqlen), d))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    rc = lib.fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                           _tok_strides(q, k, v, o, dout, dq, dk, dv), _ptr(cu_seqlens), _ptr(seqused), B, H,
                           int(max_seqlen), T, d, float(scale), int(bool(causal)), float(dropout_p), int(seed),
                           _ptr(workspace), int(workspace.numel() * workspace.element_size()), _stream(stream))
    _call(rc, "fa_bwd_varlen")
    return dq, dk, dv


def fwd_partial(q, k_win, v_win, kv_begin, causal=False, scale=None, dropout_p=0.0, seed=0, part_o=None,
                part_lse=None, stream=None):
    """The softmax piece over the key window [kv_begin, kv_begin + len) of
    every query row via ``fa_fwd_partial``: q dense [B,H,N,d]; k_win, v_win
    dense [B,H,len,d] holding those key rows.  Returns (part_o fp32
    [B,H,N,d], part_lse fp32 [B,H,N])."""
    _check_inputs(q)
    _check_dense(q, k_win, v_win)
    B, H, N, d = q.shape
    nk = k_win.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if part_o is None:
        part_o = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if part_lse is None:
        part_lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = load().fa_fwd_partial(_ptr(q), _ptr(k_win), _ptr(v_win), _ptr(part_o), _ptr(part_lse), B, H, N, d,
                               float(scale), int(bool(causal)), float(dropout_p), int(seed), int(kv_begin),
                               int(kv_begin + nk), _stream(stream))
    _call(rc, "fa_fwd_partial")
    return part_o, part_lse


def merge_partials(part_o, part_lse, o=None, lse=None, stream=None):
    """O (bf16) and lse from stacked softmax pieces part_o [S,B,H,N,d] and
    part_lse [S,B,H,N] via ``fa_merge_partials``."""
    S, B, H, N, d = part_o.shape
    if part_o.dtype != torch.float32 or part_lse.dtype != torch.float32:
        raise ValueError("partials are fp32")
    if not (part_o.is_contiguous() and part_lse.is_contiguous()) or tuple(part_lse.shape) != (S, B, H, N):
        raise ValueError("partials must be dense [S,B,H,N,d] and [S,B,H,N]")
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=part_o.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=part_o.device)
    rc = load().fa_merge_partials(_ptr(part_o), _ptr(part_lse), S, _ptr(o), _ptr(lse), B, H, N, d, _stream(stream))
    _call(rc, "fa_merge_partials")
    return o, lse


def weight_partial(part_o, all_lse, part, lse=None, stream=None):
    """``fa_weight_partial``: rescale the piece part_o (fp32 [B,H,N,d], in
    place) to e^(lse_part - lse) O_part given every piece's logsumexp all_lse
    (fp32 [S,B,H,N]); returns (part_o, lse) with lse = ln sum_s e^lse_s."""
    S = all_lse.shape[0]
    B, H, N, d = part_o.shape
    if part_o.dtype != torch.float32 or all_lse.dtype != torch.float32:
        raise ValueError("pieces are fp32")
    if not (part_o.is_contiguous() and all_lse.is_contiguous()) or tuple(all_lse.shape) != (S, B, H, N):
        raise ValueError("part_o must be dense [B,H,N,d] and all_lse dense [S,B,H,N]")
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=part_o.device)
    rc = load().fa_weight_partial(_ptr(part_o), _ptr(all_lse), S, int(part), _ptr(lse), B, H, N, d, _stream(stream))
    _call(rc, "fa_weight_partial")
    return part_o, lse


def dq_accumulator_bytes(B, H, N, d) -> int:
    return int(load().fa_bwd_dq_accumulator_bytes(B, H, N, d))


def bwd_prepare(o, dout, lse, workspace, stream=None):
    """``fa_bwd_prepare`` on dense tensors (D, scaled lse, zeroed dQ accumulator)."""
    _check_inputs(o, dout)
    _check_dense(o, dout)
    B, H, N, d = o.shape
    _call(load().fa_bwd_prepare(_ptr(o), _ptr(dout), _ptr(lse), B, H, N, d, _ptr(workspace),
                                int(workspace.numel() * workspace.element_size()), _stream(stream)), "fa_bwd_prepare")


def bwd_recompute_range(q, k_win, v_win, dout, kv_begin, workspace, causal=False, scale=None, dropout_p=0.0, seed=0,
                        dk=None, dv=None, stream=None):
    """dK, dV of the key window and its dQ part (added into the workspace's
    accumulator) via ``fa_bwd_recompute_range``."""
    _check_inputs(q, dout)
    _check_dense(q, dout, k_win, v_win)
    B, H, N, d = q.shape
    nk = k_win.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dk = torch.empty_like(k_win) if dk is None else dk
    dv = torch.empty_like(v_win) if dv is None else dv
    rc = load().fa_bwd_recompute_range(_ptr(q), _ptr(k_win), _ptr(v_win), _ptr(dout), _ptr(dk), _ptr(dv), B, H, N, d,
                                       float(scale), int(bool(causal)), float(dropout_p), int(seed), int(kv_begin),
                                       int(kv_begin + nk), _ptr(workspace),
                                       int(workspace.numel() * workspace.element_size()), _stream(stream))
    _call(rc, "fa_bwd_recompute_range")
    return dk, dv


def bwd_finalize(dq, workspace, scale, stream=None):
    """``fa_bwd_finalize``: dq = scale * the workspace accumulator, bf16."""
    _check_inputs(dq)
    _check_dense(dq)
    B, H, N, d = dq.shape
    _call(load().fa_bwd_finalize(_ptr(dq), B, H, N, d, float(scale), _ptr(workspace),
                                 int(workspace.numel() * workspace.element_size()), _stream(stream)),
          "fa_bwd_finalize")
    return dq


def dropout_mask(B, H, N, dropout_p, seed, heads, rows, device="cuda", stream=None):
    """Keep bits [nheads, nrows, N] (uint8) from the device hash."""
    h = torch.as_tensor(heads, dtype=torch.int32, device=device).contiguous()
    r = torch.as_tensor(rows, dtype=torch.int32, device=device).contiguous()
    out = torch.empty((h.numel(), r.numel(), N), dtype=torch.uint8, device=device)
    rc = load().fa_dropout_mask(B, H, N, float(dropout_p), int(seed), _ptr(h), h.numel(), _ptr(r),
                                r.numel(), _ptr(out), _stream(stream))
    _call(rc, "fa_dropout_mask")
    return out


def debug_fwd_timeout(q, k, v, causal=False, scale=None, stream=None) -> int:
    """Run ``fa_debug_fwd_timeout`` (fault injection: a forward whose first
    bounded wait runs out); returns the launch status.  Read the outcome with
    ``device_error``."""
    _check_inputs(q, k, v)
    _check_dense(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    return int(load().fa_debug_fwd_timeout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                           int(bool(causal)), _stream(stream)))


def debug_exp2_poly(x, stream=None):
    """2^x through the kernels' polynomial exponential (``fa_debug_exp2_poly``),
    for tests; x is a float32 CUDA tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    _call(load().fa_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "fa_debug_exp2_poly")
    return y


def device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the kernels' error word."""
    return int(load().fa_get_device_error(_stream(stream)))
