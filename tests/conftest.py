import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle


def pytest_terminal_summary(terminalreporter):
    # the parity diagnostic: worst error per element as a fraction of the
    # tolerance's scale sum_k |x w'| (the tolerance allows 2e-3 of it)
    mod = sys.modules.get("gpu_util")
    if mod is not None and mod.WORST["ratio"] > 0.0:
        terminalreporter.write_line(
            f"parity: max |y - y_ref| / sum|x w'| = {mod.WORST['ratio']:.3e} ({mod.WORST['what']}); "
            f"largest share of the tolerance 2e-3 sum|x w'| + 2^-8 |y| + 1e-3 used = "
            f"{mod.WORST['used']:.3f} ({mod.WORST['used_what']})")
