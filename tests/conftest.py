import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def pytest_collection_modifyitems(config, items):
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


@pytest.fixture(autouse=True, scope="session")
def _canary_guards():
    """On a GPU, every output the library writes in the tests sits between canary guard bands
    that are checked after the call (tests/guards.py)."""
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        from gated_delta_rule_62_b200 import kda as K
        from tests import guards
        guards.install(K)
    yield


def pytest_terminal_summary(terminalreporter):
    try:
        from tests import guards
    except Exception:  # pragma: no cover
        return
    if guards.checks():
        terminalreporter.write_line(f"canary guard bands checked intact: {guards.checks()}")
