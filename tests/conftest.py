import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: large oracle work (minutes of CPU)")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_sessionfinish(session, exitstatus):
    mod = sys.modules.get("oracle_pool")
    if mod is not None:
        mod.close_pool()


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the error figures of every whole-tensor oracle comparison."""
    mod = sys.modules.get("oracle_pool")
    if mod is None or not mod.SUMMARY:
        return
    terminalreporter.write_sep("-", "whole-tensor parity against the fp64 oracle")
    for r in mod.SUMMARY:
        terminalreporter.write_line(
            f"{r['name']}: {r['values']} values, out max|err| {r['out_max']:.3g} "
            f"mean {r['out_mean']:.3g}, lse max|err| {r['lse_max']:.3g}")
