import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_sessionstart(session):
    # Rebuild the CUDA library if a source is newer than it (no-op otherwise).
    from mixture_experts_layer_30_b200 import build
    build.build()


def pytest_terminal_summary(terminalreporter):
    # Router probability errors measured by the GPU parity checks.
    try:
        from tests import parity
    except Exception:
        return
    if not parity.ROUTER_ERRORS:
        return
    tr = terminalreporter
    tr.section("router probability error vs the fp64 oracle")
    tr.write_line(f"{'forward pass':<36} {'max |dp|':>10} {'at the decision boundary':>26}")
    for label, (e_all, e_bd) in sorted(parity.ROUTER_ERRORS.items()):
        tr.write_line(f"{label:<36} {e_all:>10.3g} {e_bd:>26.3g}")
