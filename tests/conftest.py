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
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


# The parity tests print one "[parity] ..." line per compared case (the measured
# max |y - y_ref| / (1 + |y_ref|)); pytest captures the output of passing tests,
# so the lines are collected here and repeated in the session summary.
_PARITY_LINES = []


def pytest_runtest_logreport(report):
    if report.when == "call" and report.passed:
        for line in report.capstdout.splitlines():
            if line.startswith("[parity]"):
                _PARITY_LINES.append(line)


def pytest_terminal_summary(terminalreporter):
    if _PARITY_LINES:
        terminalreporter.write_sep("-", "measured parity errors, max |y - y_ref| / (1 + |y_ref|)")
        for line in _PARITY_LINES:
            terminalreporter.write_line(line)
