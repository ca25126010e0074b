import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU-only oracle checks")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Worst parity error each test reached against its bar (max-abs on the float32
    path, per-(sequence, head) relative L2 on the bf16 path)."""
    try:
        from tests import _parity as P
    except Exception:  # pragma: no cover
        return
    if not P.MARGINS:
        return
    worst = {}
    for test, what, kind, err, bar in P.MARGINS:
        key = (test, what, kind)
        if key not in worst or err / bar > worst[key][0] / worst[key][1]:
            worst[key] = (err, bar)
    terminalreporter.section("parity margins (worst per test; error / bar)")
    for (test, what, kind), (err, bar) in sorted(worst.items()):
        terminalreporter.write_line(f"{err:10.3e} / {bar:.0e}  {kind:16s} {what:28s} {test}")
