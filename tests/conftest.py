import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def lib():
    """The built C-ABI library (built on demand; no GPU needed to load it)."""
    from persistent_sm_attn_b200 import binding
    return binding.load()


def pytest_terminal_summary(terminalreporter):
    """Print the relative Frobenius errors the GPU parity tests measured."""
    gu = sys.modules.get("tests.gpu_util")
    if gu is None or not getattr(gu, "MARGINS", None):
        return
    terminalreporter.section("parity margins (relative Frobenius error, bound 5e-3)")
    for label, errs in gu.MARGINS:
        terminalreporter.write_line(
            f"{label:<64} " + "  ".join(f"{k} {v:.3e}" for k, v in errs.items()))
