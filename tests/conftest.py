import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Max scaled error |gpu - oracle| / (1 + |oracle|) of every GPU parity
    comparison in this session, against its tolerance."""
    mod = sys.modules.get("test_gpu_parity") or sys.modules.get("tests.test_gpu_parity")
    rows = list(getattr(mod, "ERRORS", [])) if mod else []
    for name in ("test_gpu_forgetting", "tests.test_gpu_forgetting"):
        m = sys.modules.get(name)
        if m is not None and getattr(m, "ERRORS", None) is not None and m.ERRORS is not rows:
            rows += [r for r in m.ERRORS if r not in rows]
    if not rows:
        return
    terminalreporter.write_sep("-", "max scaled error per comparison (gpu vs oracle)")
    for test, what, err, tol in rows:
        terminalreporter.write_line("%-60s %-22s %.3e  (tol %.0e, headroom %.0fx)" % (
            test[:60], what[:22], err, tol, tol / err if err > 0 else float("inf")))
