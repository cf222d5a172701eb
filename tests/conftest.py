import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle.lib()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Report how many compared outputs used the one-bf16-step allowance of
    the parity bar (reading C11), per comparison that used it."""
    mod = sys.modules.get("tests._gpu_util")
    if mod is None or not getattr(mod, "STEP_LOG", None):
        return
    used = [(lab, n, m) for (lab, n, m) in mod.STEP_LOG if n]
    total = sum(m for (_, _, m) in mod.STEP_LOG)
    terminalreporter.write_line(
        f"parity: {len(mod.STEP_LOG)} comparisons, {total} elements; "
        f"{sum(n for (_, n, _) in used)} used the one-bf16-step allowance")
    for lab, n, m in used:
        terminalreporter.write_line(f"  {lab or '(unlabelled)'}: {n} of {m}")
