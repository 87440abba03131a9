import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")
    config.addinivalue_line(
        "markers", "slow: long CPU test (oracle at full workload size)")
    config.addinivalue_line(
        "markers", "last: run after every other collected test (newest GPU paths)")


def pytest_collection_modifyitems(config, items):
    """Tests marked ``last`` run after all others, in their collected order,
    so that a run stopping at the first failure has already run the rest."""
    items[:] = ([it for it in items if it.get_closest_marker("last") is None]
                + [it for it in items if it.get_closest_marker("last") is not None])


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library binding; a GPU test must never fall back to anything."""
    if not gpu_available():
        pytest.fail("a test marked gpu ran without a CUDA device")
    from gated_delta_rule_114_b200 import ckda
    ckda.load()
    return ckda


def pytest_terminal_summary(terminalreporter):
    """Print the literal max|x - x_ref| / rms(x_ref) of every parity check the
    session ran (the largest per test and output; step numbers folded), next
    to its bound, so a passing run shows its margins."""
    import re
    try:
        from parity_util import RECORDED
    except ImportError:
        return
    if not RECORDED:
        return
    worst = {}
    for test_id, what, ratio, rel, store in RECORDED:
        key = (test_id, re.sub(r"\d+", "#", what))
        if key not in worst or ratio > worst[key][0]:
            worst[key] = (ratio, rel, store)
    tr = terminalreporter
    tr.section("parity margins: literal max|x - x_ref| / rms(x_ref)")
    for (test_id, what), (ratio, rel, store) in worst.items():
        allow = "%.0e rms" % rel + (" + 2^-8|x_ref|" if store else "")
        tr.write_line("%-9.3e  (bound %s)  %s  [%s]" % (ratio, allow, test_id, what))
