import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


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


@pytest.fixture(autouse=True, scope="session")
def _short_device_waits():
    """GPU tests run with a 500 ms limit on every device-side wait (the library
    default is 2 s), so that a broken pipeline gives up quickly."""
    try:
        import torch
        if torch.cuda.is_available():
            from long_context_attention_fwd_b200 import capi
            capi.attn_set_wait_timeout_ns(500_000_000)
    except Exception:
        pass
    yield


def pytest_terminal_summary(terminalreporter):
    """Prints the parity figures the GPU tests recorded (strict O counts, gradient
    errors), so that a run's output shows them whether the tests passed or not."""
    try:
        from helpers import PARITY_LOG
    except Exception:
        return
    if not PARITY_LOG:
        return
    import json
    terminalreporter.section("parity figures")
    for label, metrics in PARITY_LOG:
        terminalreporter.write_line(f"{label}: {json.dumps(metrics, sort_keys=True)}")
