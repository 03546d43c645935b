"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Plugin or custom-op interfaces that pass a kernel only its inputs and
outputs, or code that must not allocate at that point, have no way to give
fa_bwd a workspace; fa_bwd_noalloc takes its scratch from a static array in
the library instead.  This file checks it through the C ABI against fa_bwd on
the same inputs, on two calls in a row (the second call finds the first
call's leftovers in the shared scratch), and that shapes beyond the scratch
limit are refused.  It is named so that pytest collects it last.
"""
import math

import pytest
import torch

from io_aware_exact_25_b200 import binding
from io_aware_exact_25_b200.inputs import make_inputs

MAX_ABS = 2e-2
REL_L2 = 5e-3


def _close(a, b, what):
    a, b = a.float(), b.float()
    err = (a - b).abs().max().item()
    rel = ((a - b).norm() / b.norm().clamp_min(1e-30)).item()
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max abs {err:.3e}, rel L2 {rel:.3e}"


@pytest.mark.gpu
@pytest.mark.parametrize("causal,p,d", [(True, 0.0, 128), (False, 0.1, 64)])
def test_noalloc_backward_matches_fa_bwd_on_two_calls(cuda_device, causal, p, d):
    B, H, N = 1, 3, 700
    assert binding.bwd_workspace_size(B, H, N, d) <= binding.NOALLOC_SCRATCH_BYTES
    x = {n: t.to(cuda_device) for n, t in make_inputs(B, H, N, d, seed=77).items()}
    scale = 1.0 / math.sqrt(d)
    o, lse = binding.fwd(x["q"], x["k"], x["v"], causal=causal, scale=scale, dropout_p=p, seed=5)
    ref = binding.bwd(x["q"], x["k"], x["v"], o, x["do"], lse, causal=causal, scale=scale, dropout_p=p, seed=5)
    for call in range(2):
        out = [torch.full_like(x["q"], float("nan")) for _ in range(3)]
        binding.bwd_noalloc(x["q"], x["k"], x["v"], o, x["do"], lse, *out, causal=causal, scale=scale,
                            dropout_p=p, seed=5)
        torch.cuda.synchronize()
        assert binding.device_error() == 0
        for name, got, want in zip(("dQ", "dK", "dV"), out, ref):
            _close(got, want, f"call {call} {name}")


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_the_scratch(cuda_device):
    B, H, N, d = 4, 16, 2048, 128  # needs 64 MiB + row vectors of scratch
    assert binding.bwd_workspace_size(B, H, N, d) > binding.NOALLOC_SCRATCH_BYTES
    lib = binding.load()
    rc = lib.fa_bwd_noalloc(16, 16, 16, 16, 16, 16, 16, 16, 16, B, H, N, d, 0.1, 1, 0.0, 0, None)
    assert rc == binding.FA_ERR_TOO_LARGE
