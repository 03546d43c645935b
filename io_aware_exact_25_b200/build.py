"""Build the C-ABI library in-tree with nvcc for sm_100a: ``libfa_sm100.so``
(release) and ``libfa_sm100_debug.so`` (the bounds-checking build, FA_DEBUG)."""
from __future__ import annotations

import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libfa_sm100.so")
DEBUG_LIB = os.path.join(PKG, "libfa_sm100_debug.so")
SOURCES = [os.path.join(PKG, "csrc", n) for n in ("fa_api.cu", "fa_noalloc.cu", "fa_seqpar.cu")]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", "-shared"]


def _inputs() -> list:
    return (glob.glob(os.path.join(PKG, "csrc", "*")) + [os.path.join(ROOT, "include", "fa.h"),
                                                          os.path.abspath(__file__)])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def _compile(lib: str, extra: list, verbose: bool) -> None:
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Compile the release library (and, with ``debug``, the bounds-checking
    one) if a source changed since; returns the release library's path."""
    if force or not up_to_date(LIB):
        _compile(LIB, [], verbose)
    if debug and (force or not up_to_date(DEBUG_LIB)):
        _compile(DEBUG_LIB, ["-DFA_DEBUG"], False)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
