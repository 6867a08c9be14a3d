import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_terminal_summary(terminalreporter):
    """Element-wise error diagnostic of every CUDA-vs-oracle comparison made in
    this session: the 12 worst figures, and every comparison of the full-size
    workloads (sampled heads, final decode state)."""
    from tests.parity import REPORT
    if not REPORT:
        return
    tr = terminalreporter
    tr.section("parity: element-wise error diagnostic (reported, not enforced)")
    tr.write_line(f"{len(REPORT)} comparisons; element-wise = max|x-r| / (|r| + 1e-3 rms(r))")
    tr.write_line(f"{'comparison':60s} {'max rel err':>12s} {'element-wise':>12s}")
    worst = sorted(REPORT, key=lambda r: -r[2])[:12]
    for what, e, d in worst:
        tr.write_line(f"{what[:60]:60s} {e:12.3e} {d:12.3e}")
    full = [r for r in REPORT if r[0].startswith(("head", "workload", "config 4"))]
    if full:
        tr.write_line("-- full-size workloads --")
        for what, e, d in full:
            tr.write_line(f"{what[:60]:60s} {e:12.3e} {d:12.3e}")
