import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size shapes (seconds to minutes)")


@pytest.fixture(scope="session", autouse=True)
def _host_generator():
    """The C host fill of the seeded generator (same bits as numpy, much faster)."""
    import synth
    synth.build_host_fill()


@pytest.fixture(scope="session")
def oracle_ref():
    import oracle
    oracle.build()
    return oracle.Oracle()


def pytest_terminal_summary(terminalreporter):
    """Worst errors the parity checks met (against their tolerances), when any ran."""
    import sys
    h = sys.modules.get("tests.harness")
    if h is not None and h.WORST["out_excess"] > -1.0:
        w = h.WORST
        terminalreporter.write_line(
            f"parity worst: gate |err| {w['gate_abs']:.3g} (tol {h.GATE_ATOL:g}), logit |err| "
            f"{w['logit_abs']:.3g}, output excess over tolerance {w['out_excess']:.3g}, "
            f"rel L2 {w['out_rel_l2']:.3g} (tol {h.REL_L2:g})")
