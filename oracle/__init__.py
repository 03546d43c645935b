"""Test infrastructure: the fp64 CPU oracle for exact attention.

This package is NOT part of the product.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg import it.
It wraps ``attention_oracle.c`` (plain C, fp64, OpenMP over rows) through
ctypes and takes inputs as bf16 bit patterns (``numpy.uint16`` arrays of shape
``[B, H, N, d]``, or torch bf16 tensors), so the oracle sees exactly the
values the GPU sees.  float64 inputs are accepted too, for the
finite-difference pins.

What each function computes, and the passages it follows, is documented in
the C source.  Every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, invariants, finite differences and torch's fp64 CPU
``scaled_dot_product_attention``; the dropout hash beyond its statistical
properties and published constants is this library's own definition.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` with gcc (-O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # ORACLE_LIB points the pins at another build of the same source (the
        # mutation test compiles deliberately broken copies to prove the pins
        # catch them).
        lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        vp = ctypes.c_void_p
        i32p = ctypes.POINTER(ctypes.c_int32)
        f64p = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        I, D, U64 = ctypes.c_int, ctypes.c_double, ctypes.c_uint64
        lib.orc_forward.argtypes = [vp, vp, vp, I, I, I, I, I, D, I, D, U64,
                                    i32p, I, i32p, I, f64p, f64p]
        lib.orc_backward_q.argtypes = [vp, vp, vp, vp, I, I, I, I, I, D, I, D, U64,
                                       i32p, I, i32p, I, f64p, f64p, f64p]
        lib.orc_backward_kv.argtypes = [vp, vp, vp, vp, I, I, I, I, I, D, I, D, U64,
                                        i32p, I, i32p, I, f64p, f64p]
        lib.orc_dropout_mask.argtypes = [I, I, I, D, U64, i32p, I, i32p, I, u8p]
        for fn in (lib.orc_forward, lib.orc_backward_q, lib.orc_backward_kv, lib.orc_dropout_mask):
            fn.restype = ctypes.c_int
        lib.orc_hash32.argtypes = [U64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
                                   ctypes.c_uint32]
        lib.orc_hash32.restype = ctypes.c_uint32
        lib.orc_keep_threshold.argtypes = [D]
        lib.orc_keep_threshold.restype = ctypes.c_uint32
        lib.orc_hash_constant.argtypes = [I]
        lib.orc_hash_constant.restype = ctypes.c_uint32
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_set_block_mask.argtypes = [u8p, I, I]
        lib.orc_set_block_mask.restype = None
        lib.orc_set_seqlens.argtypes = [i32p]
        lib.orc_set_seqlens.restype = None
        _lib = lib
        return lib


def _bits(t) -> np.ndarray:
    """C-contiguous input array: bf16 bit patterns (uint16) or float64.

    torch bf16 tensors become their uint16 bit patterns; torch float64 tensors
    become float64 arrays.  Any other dtype is refused.
    """
    if not isinstance(t, np.ndarray):  # torch tensor
        import torch
        t = t.detach().to("cpu").contiguous()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16).numpy().view(np.uint16)
        elif t.dtype == torch.float64:
            t = t.numpy()
        else:
            raise TypeError("oracle inputs are bf16 or float64")
    if t.dtype not in (np.uint16, np.float64):
        raise TypeError("oracle inputs are bf16 bit patterns (uint16) or float64")
    return np.ascontiguousarray(t)


def _kind(*arrays) -> int:
    """1 if the inputs are float64, 0 if bf16 bit patterns; they must agree."""
    kinds = {a.dtype for a in arrays}
    if len(kinds) != 1:
        raise TypeError("oracle inputs must share one dtype")
    shapes = {a.shape for a in arrays}
    if len(shapes) != 1 or len(arrays[0].shape) != 4:
        raise ValueError("oracle inputs must share one [B,H,N,d] shape")
    return int(arrays[0].dtype == np.float64)


def _idx(sel, default_n):
    if sel is None:
        return None, default_n
    a = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    return a, int(a.size)


def _p(a, ctype):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctype))


class _SeqLens:
    """Installs per-batch sequence lengths for the oracle calls made inside
    the ``with``: rows and keys at or beyond ``seqlens[b]`` of batch entry b
    are padding ("FlashAttention for Efficient Training", section 5.2:
    A_ij = -inf unless the key lies within the sequence).  Padding queries
    get O = 0, lse = -inf and dQ = 0; padding keys get dK = dV = 0."""

    def __init__(self, seqlens, B, N):
        self.arr = None
        if seqlens is None:
            return
        a = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int64))
        if a.shape != (B,) or (a < 0).any() or (a > N).any():
            raise ValueError(f"seqlens must be {B} lengths in [0, {N}], got {a.tolist()}")
        self.arr = a.astype(np.int32)

    def __enter__(self):
        if self.arr is not None:
            _load().orc_set_seqlens(_p(self.arr, ctypes.c_int32))
        return self

    def __exit__(self, *exc):
        if self.arr is not None:
            _load().orc_set_seqlens(None)
        return False


class _BlockMask:
    """Installs a block mask for the oracle calls made inside the ``with``.

    ``mask`` is ``[heads, nt, nt]`` with heads 1 (shared by every head) or H
    and ``nt = ceil(N / tile)``; a zero at ``[h, a, c]`` hides keys of tile c
    from queries of tile a.  The C side keeps the pointer per thread, so the
    array is held here until the call returns.
    """

    def __init__(self, mask, H, N, tile):
        self.arr = None
        if mask is None:
            return
        if not isinstance(mask, np.ndarray):
            mask = mask.detach().to("cpu").numpy()
        a = np.ascontiguousarray(np.asarray(mask) != 0, dtype=np.uint8)
        nt = (N + tile - 1) // tile
        if a.ndim != 3 or a.shape[0] not in (1, H) or a.shape[1:] != (nt, nt):
            raise ValueError(f"block mask must be [1 or H, {nt}, {nt}], got {a.shape}")
        self.arr, self.tile = a, int(tile)

    def __enter__(self):
        if self.arr is not None:
            _load().orc_set_block_mask(_p(self.arr, ctypes.c_uint8), self.arr.shape[0], self.tile)
        return self

    def __exit__(self, *exc):
        if self.arr is not None:
            _load().orc_set_block_mask(None, 1, 128)
        return False


def num_threads() -> int:
    """OpenMP threads the oracle uses (``OMP_NUM_THREADS`` or all cores)."""
    return int(_load().orc_num_threads())


def forward(q, k, v, scale, causal=False, p_drop=0.0, seed=0, heads=None, rows=None,
            block_mask=None, block=128, seqlens=None):
    """O_i and lse_i for the selected heads (bh = b*H + h) and query rows.

    Returns ``(o, lse)`` as float64 arrays of shape ``[nheads, nrows, d]`` and
    ``[nheads, nrows]``.  ``block_mask`` (``[1 or H, nt, nt]`` over
    ``block``-sized tiles) hides whole key tiles; a row that sees no key gets
    O = 0 and lse = -inf.  ``seqlens`` (``[B]``) marks rows and keys at or
    beyond ``seqlens[b]`` of batch entry b as padding.
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    f64 = _kind(qb, kb, vb)
    B, H, N, d = qb.shape
    hs, nh = _idx(heads, B * H)
    rs, nr = _idx(rows, N)
    o = np.empty((nh, nr, d), np.float64)
    lse = np.empty((nh, nr), np.float64)
    with _BlockMask(block_mask, H, N, block), _SeqLens(seqlens, B, N):
        rc = _load().orc_forward(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, f64,
                                 B, H, N, d, float(scale), int(bool(causal)), float(p_drop), int(seed),
                                 _p(hs, ctypes.c_int32), nh, _p(rs, ctypes.c_int32), nr,
                                 _p(o, ctypes.c_double), _p(lse, ctypes.c_double))
    if rc:
        raise RuntimeError(f"orc_forward failed ({rc})")
    return o, lse


def backward_q(q, k, v, dout, scale, causal=False, p_drop=0.0, seed=0, heads=None, rows=None,
               block_mask=None, block=128, seqlens=None):
    """dQ_i and D_i for the selected query rows.

    Returns ``(dq, D, max_rel_dev)``; ``max_rel_dev`` is the largest relative
    gap between D_i = sum_j P_ij dP_ij and <dO_i, O_i> (they are equal in
    exact arithmetic).
    """
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    f64 = _kind(qb, kb, vb, db)
    B, H, N, d = qb.shape
    hs, nh = _idx(heads, B * H)
    rs, nr = _idx(rows, N)
    dq = np.empty((nh, nr, d), np.float64)
    D = np.empty((nh, nr), np.float64)
    dev = ctypes.c_double(0.0)
    with _BlockMask(block_mask, H, N, block), _SeqLens(seqlens, B, N):
        rc = _load().orc_backward_q(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
                                    db.ctypes.data, f64, B, H, N, d, float(scale), int(bool(causal)),
                                    float(p_drop), int(seed), _p(hs, ctypes.c_int32), nh,
                                    _p(rs, ctypes.c_int32), nr, _p(dq, ctypes.c_double),
                                    _p(D, ctypes.c_double), ctypes.byref(dev))
    if rc:
        raise RuntimeError(f"orc_backward_q failed ({rc})")
    return dq, D, dev.value


def backward_kv(q, k, v, dout, scale, causal=False, p_drop=0.0, seed=0, heads=None, keys=None,
                block_mask=None, block=128, seqlens=None):
    """dK_j and dV_j for the selected heads and key rows.

    Returns ``(dk, dv)`` of shape ``[nheads, nkeys, d]``.
    """
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    f64 = _kind(qb, kb, vb, db)
    B, H, N, d = qb.shape
    hs, nh = _idx(heads, B * H)
    ks, nk = _idx(keys, N)
    dk = np.empty((nh, nk, d), np.float64)
    dv = np.empty((nh, nk, d), np.float64)
    with _BlockMask(block_mask, H, N, block), _SeqLens(seqlens, B, N):
        rc = _load().orc_backward_kv(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
                                     db.ctypes.data, f64, B, H, N, d, float(scale), int(bool(causal)),
                                     float(p_drop), int(seed), _p(hs, ctypes.c_int32), nh,
                                     _p(ks, ctypes.c_int32), nk, _p(dk, ctypes.c_double),
                                     _p(dv, ctypes.c_double))
    if rc:
        raise RuntimeError(f"orc_backward_kv failed ({rc})")
    return dk, dv


def dropout_mask(B, H, N, p_drop, seed, heads=None, rows=None) -> np.ndarray:
    """Keep bits Z_ij (1 = kept) as uint8 ``[nheads, nrows, N]``."""
    hs, nh = _idx(heads, B * H)
    rs, nr = _idx(rows, N)
    out = np.empty((nh, nr, N), np.uint8)
    rc = _load().orc_dropout_mask(B, H, N, float(p_drop), int(seed), _p(hs, ctypes.c_int32), nh,
                                  _p(rs, ctypes.c_int32), nr, _p(out, ctypes.c_uint8))
    if rc:
        raise RuntimeError(f"orc_dropout_mask failed ({rc})")
    return out


def hash32(seed, b, h, i, j) -> int:
    return int(_load().orc_hash32(int(seed), int(b), int(h), int(i), int(j)))


def keep_threshold(p_drop) -> int:
    return int(_load().orc_keep_threshold(float(p_drop)))


def hash_constants() -> tuple[int, int, int]:
    """(C1, C2, G) as the oracle derives them."""
    lib = _load()
    return tuple(int(lib.orc_hash_constant(w)) for w in range(3))
