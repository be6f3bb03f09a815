import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Worst gradient ratios |g - g_ref| / (rtol |g_ref| + m S) of the GPU
    parity checks, at each recorded floor m."""
    try:
        from tests.gpu_helpers import FLOORS, GRAD_RATIOS
    except Exception:
        return
    if not GRAD_RATIOS:
        return
    tr = terminalreporter
    tr.write_sep("-", "gradient parity: worst ratio per check (<= 1 passes)")
    tr.write_line(f"{'check':60s} {'elements':>10s} {'rtol':>7s} " + " ".join(f"{'m=%g' % m:>10s}" for m in FLOORS))
    for what, n, rtol, worst in GRAD_RATIOS:
        tr.write_line(f"{what[:60]:60s} {n:10d} {rtol:7.0e} " + " ".join(f"{w:10.4f}" for w in worst))
    tr.write_line("overall worst: " + ", ".join(f"m={m:g}: {max(r[3][k] for r in GRAD_RATIOS):.4f}"
                                                for k, m in enumerate(FLOORS)))


def pytest_sessionfinish(session, exitstatus):
    """Under GS_CHECKED=1 (the bounds-checked library) a session that ran GPU
    tests fails if any device-side check fired."""
    if os.environ.get("GS_CHECKED") != "1":
        return
    try:
        import torch
        if not torch.cuda.is_available():
            return
        from differentiable_tile_rasterizer_b200 import gs
        if gs._LIB is None:
            return
        assert gs.gs_debug_is_checked_build(), "GS_CHECKED=1 but the unchecked library is loaded"
        st = gs.gs_debug_checked_status()
    except Exception as e:  # report, do not mask the tests' own status
        print(f"\nchecked build: status not read ({e})")
        session.exitstatus = 1
        return
    print(f"\nchecked build: device-side check status {st}")
    if st != 0:
        session.exitstatus = 1
