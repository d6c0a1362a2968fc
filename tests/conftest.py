import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def lib():
    """The CUDA library, built in-tree; GPU tests fail loudly if it is missing."""
    from nvfp4_block_scaled_15_b200 import nvfp4
    return nvfp4


def pytest_terminal_summary(terminalreporter):
    """Per test: bf16 outputs that passed only by the carried pre-cast bound."""
    parity = sys.modules.get("parity")
    log = getattr(parity, "CARRIED_LOG", None) if parity else None
    if not log:
        return
    per = {}
    for test, n, size in log:
        c, t = per.get(test, (0, 0))
        per[test] = (c + n, t + size)
    total_c = sum(c for c, _ in per.values())
    total_t = sum(t for _, t in per.values())
    terminalreporter.write_sep("-", "bf16 outputs passing only by the carried pre-cast bound")
    for test, (c, t) in sorted(per.items()):
        if c:
            terminalreporter.write_line(f"{test}: {c} of {t}")
    terminalreporter.write_line(f"all bf16 checks: {total_c} of {total_t} outputs ({len(per)} tests)")
