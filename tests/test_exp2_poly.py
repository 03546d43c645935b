"""The polynomial exponential of the backward kernel's probabilities.

2^x = 2^n * 2^f with n = round(x) and f in [-1/2, 1/2] (Cody-Waite range
reduction), 2^f from a cubic fitted for minimal relative error on
[-1/2, 1/2] (Remez exchange).  The CPU tests read the cubic's coefficients
from the kernel source and hold them to what a minimax fit must satisfy; the
GPU test runs the device function itself (``fa_debug_exp2_poly``) against
CUDA's exp2 and the exact value.
"""
import math
import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "..", "io_aware_exact_25_b200", "csrc", "sm100.cuh")
BOUND = 7.5e-5  # the maximum relative error the kernel source states for its cubic


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("void exp2_poly_x2"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([-0-9.e]+)f, \1f\)", body)]
    # the four Horner constants, highest degree first (after the rounding constants and -1)
    coef = [v for v in vals if abs(v) < 2.0 and v != -1.0]
    assert len(coef) == 4, coef
    return [float(np.float32(c)) for c in coef]


def _rel_err(f):
    c3, c2, c1, c0 = _coefficients()
    p = ((c3 * f + c2) * f + c1) * f + c0
    return p / np.exp2(f) - 1.0


def test_cubic_meets_its_bound_on_the_reduced_range():
    f = np.linspace(-0.5, 0.5, 200001)
    assert np.max(np.abs(_rel_err(f))) <= BOUND * 1.01


def test_cubic_equioscillates():
    """A minimax cubic's error takes its maximum magnitude at 5 points with
    alternating signs (Chebyshev's alternation theorem): a Taylor cubic or a
    least-squares fit does not, and a wrong coefficient breaks it."""
    f = np.linspace(-0.5, 0.5, 200001)
    e = _rel_err(f)
    emax = np.max(np.abs(e))
    # local extrema of e including the interval ends
    idx = [0] + [i for i in range(1, len(e) - 1) if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0] + [len(e) - 1]
    ext = [e[i] for i in idx if abs(e[i]) >= 0.9 * emax]
    signs = np.sign(ext)
    assert len(ext) >= 5
    assert all(signs[i] != signs[i + 1] for i in range(len(signs) - 1))


def test_reduction_splits_exactly():
    """x - round(x) by adding and subtracting 1.5 * 2^23 is exact in fp32 for
    |x| <= 126 and lands in [-1/2, 1/2]."""
    x = np.float32(np.random.default_rng(0).uniform(-126, 126, 100000))
    magic = np.float32(12582912.0)
    n = (x + magic) - magic
    fr = x - n
    assert np.all(np.abs(fr) <= 0.5)
    assert np.array_equal(n.astype(np.float64) + fr.astype(np.float64), x.astype(np.float64))


@pytest.mark.gpu
def test_device_function_against_cuda_exp2(cuda_device):
    import torch
    from io_aware_exact_25_b200 import binding
    rng = np.random.default_rng(1)
    x = np.concatenate([np.linspace(-126.0, 126.0, 1 << 20), rng.uniform(-30.0, 0.0, 1 << 20),
                        np.arange(-126.0, 127.0), [0.0, -0.5, 0.5, -1e-30, 1e-30]]).astype(np.float32)
    xd = torch.from_numpy(x).to(cuda_device)
    y = binding.debug_exp2_poly(xd)
    cuda_ref = torch.exp2(xd)  # CUDA's single-precision exp2
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    got = y.cpu().numpy().astype(np.float64)
    # the bound holds where 2^n * 2^f is a normal float (x >= -125); below,
    # where probabilities are < 2^-125 and vanish in bf16, only 0 <= y <= 2^-124
    normal = x >= -125.0
    rel = np.abs(got[normal] / exact[normal] - 1.0)
    assert rel.max() <= BOUND * 1.05, f"max rel err {rel.max():.3e} at x={x[normal][np.argmax(rel)]}"
    rel_cuda = np.abs(got[normal] / cuda_ref.cpu().numpy().astype(np.float64)[normal] - 1.0)
    assert rel_cuda.max() <= BOUND * 1.05 + 2 * 2.0 ** -23
    assert np.all(got[~normal] >= 0.0) and np.all(got[~normal] <= 2.0 ** -124)
    # an odd count exercises the single-element tail; below -126 the result is tiny, not zero
    t = binding.debug_exp2_poly(torch.tensor([-math.inf, -1000.0, -127.5], device=cuda_device))
    assert t.shape == (3,) and bool((t >= 0).all()) and float(t.max()) <= 2.0 ** -124
    assert binding.device_error() == 0
