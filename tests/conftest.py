import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # GPU tests are only meaningful with a device; skip them cleanly elsewhere.
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


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Ties between the CUDA path and the oracle (entries inside the 1e-5 band of a threshold,
    which may go either way): one line per compared selection, and the full record as JSON
    when CRISP_TIE_LOG names a file."""
    mod = sys.modules.get("tests.parity")
    if mod is None or not mod.TIE_LOG:
        return
    terminalreporter.write_sep("-", "selection ties vs the oracle")
    for line in mod.tie_summary_lines():
        terminalreporter.write_line(line)
    path = os.environ.get("CRISP_TIE_LOG")
    if path:
        import json
        os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
        with open(path, "w") as f:
            json.dump(mod.TIE_LOG, f, indent=1)
