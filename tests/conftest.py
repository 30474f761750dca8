import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device; CPU runs select them out with -m "not gpu".
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    # Measured errors of the GPU parity comparisons (tests/gpu_helpers.assert_close).
    try:
        from tests import gpu_helpers
    except Exception:  # the GPU helpers need the library; nothing was measured then
        return
    if not gpu_helpers.MEASURED:
        return
    tr = terminalreporter
    tr.section("parity: measured errors against the oracle")
    for what, mx, rl, bar, max_bar in gpu_helpers.MEASURED:
        tr.write_line(f"{what:60s} max_abs={mx:.3e} rel_l1={rl:.3e} (bar {max_bar} / {bar:.0e})")
