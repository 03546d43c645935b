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
