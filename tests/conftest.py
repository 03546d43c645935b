import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, TESTS):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _parity_test_id(request):
    import parity
    parity.set_current_test(request.node.nodeid)
    yield


@pytest.fixture(autouse=True)
def _bounds_record(request):
    """With FA_BOUNDS_CHECK=1 the whole suite runs on the bounds-checking
    build: after every GPU test its record of failed checks must be empty."""
    yield
    if os.environ.get("FA_BOUNDS_CHECK") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from io_aware_exact_25_b200 import binding
    lib = binding.load()
    if lib.fa_debug_build() != 1:
        return  # a test swapped in another build and has not restored it
    rec = binding.debug_bounds_record()
    assert rec[0] == 0, (f"bounds check failed: site {rec[1]}, offset {rec[2]}, limit {rec[3]}, block {rec[4]}, "
                         f"thread {rec[5]} ({rec[0]} failures)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print every use of the parity bar's recorded exception (elements above
    2e-2 that the |ref| >= 4 rounding allowance admits)."""
    import parity
    recs = parity.RECORDS
    if not recs:
        return
    tr = terminalreporter
    tr.section("parity: elements above the 2e-2 bound (|ref| >= 4 rounding allowance)")
    total = sum(r["over_2e-2"] for r in recs)
    tr.write_line(f"{len(recs)} checks used it, {total} elements in all")
    for r in recs:
        tr.write_line(f"{r['test']} {r['tensor']}: {r['over_2e-2']}/{r['elements']} (cap {r['cap']}), "
                      f"worst {r['worst_err']:.4e} at ref {r['ref_at_worst']:.4f} "
                      f"(bound {r['bound_at_worst']:.4e}, scale {r['scale']:g})")
