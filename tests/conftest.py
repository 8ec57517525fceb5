import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for p in (ROOT, os.path.join(ROOT, "oracle")):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size cases (minutes)")


def has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def orc():
    import zha_oracle
    zha_oracle.build_library()
    return zha_oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report the routing boundary flips (nodes kept by the GPU or by the
    oracle only, all within the score-error band of p) that the routing
    parity tests met, with each flip's distance from p."""
    mod = sys.modules.get("zha_testlib")
    if mod is None or not mod.ROUTES_COMPARED["heads"]:
        return
    flips = mod.FLIPS
    tr = terminalreporter
    tr.section("routing boundary flips vs the oracle")
    tr.write_line(f"head routings compared: {mod.ROUTES_COMPARED['heads']}; flips: {len(flips)}"
                  + (f"; largest distance of a flip's running mass from p: {max(f['dist'] for f in flips):.3e}"
                     if flips else ""))
    for f in flips:
        tr.write_line(f"  {f['test']} group {f['group']} level {f['level']} head {f['head']} node {f['node']}: "
                      f"running mass before it {f['cum_before']:.7f}, p {f['p']}, |diff| {f['dist']:.2e} "
                      f"(band {f['band']:.2e}, near-tie mass {f['near_tie_mass']:.2e}), kept by the {f['kept_by']} only")
