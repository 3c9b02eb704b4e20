import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this environment")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Lists the elementwise relative errors the parity checks recorded (the
    bars gate the normalised max-abs error; this figure is reported only)."""
    try:
        from parity_util import REPORT
    except Exception:  # pragma: no cover
        return
    if not REPORT:
        return
    tr = terminalreporter
    tr.section("parity errors (normalised max-abs | elementwise rel., floor 1e-3 rms)")
    worst = {}
    for name, dt, e_o, e_s, r_o, r_s in REPORT:
        k = (name, dt)
        prev = worst.get(k)
        cur = (max(e_o, e_s), max(r_o, r_s))
        worst[k] = cur if prev is None else (max(prev[0], cur[0]), max(prev[1], cur[1]))
    for (name, dt), (e, r) in sorted(worst.items()):
        tr.write_line("%-34s %-5s norm %.3e  elem %.3e" % (name, dt, e, r))
