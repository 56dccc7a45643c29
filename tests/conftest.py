import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Max err/rms and the count of justified rounding flips per parity check."""
    helpers = sys.modules.get("helpers")
    rep = getattr(helpers, "REPORT", None) if helpers else None
    if not rep:
        return
    worst = max(rep, key=lambda r: r[1])
    flips = sum(r[2] for r in rep)
    terminalreporter.write_sep("-", "parity tolerance")
    terminalreporter.write_line("%d tensor checks; max err/rms %.4f (%s); %d elements beyond 2e-2*rms, each a "
                                "justified rounding flip" % (len(rep), worst[1], worst[0], flips))
    for name, ratio, n_over, n in rep:
        if n_over:
            terminalreporter.write_line("  %s: %d of %d elements flipped, max err/rms %.4f" % (name, n_over, n, ratio))
