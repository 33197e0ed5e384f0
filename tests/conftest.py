import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an sm_100a GPU and the built CUDA library")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Table of every forward parity comparison made in the session: rows
    compared, O max / mean error, the bf16 storage floor (the fp64 oracle
    rounded to bf16), the elements over 1e-2 and how many of those lie
    within their floor plus the stated slack, and the LSE error."""
    parity = sys.modules.get("parity")
    if parity is None or not hasattr(parity, "parity_records"):
        return
    recs = parity.parity_records()
    if not recs:
        return
    tr = terminalreporter
    tr.section("forward parity (fp64 oracle vs GPU)")
    tr.write_line(f"{'comparison':58s} {'rows':>8s} {'O max':>9s} {'O mean':>9s} "
                  f"{'floor max':>9s} {'>1e-2':>6s} {'in floor':>8s} {'LSE max':>9s}")

    def f(x):
        return "-" if x is None else f"{x:.2e}"

    def i(x):
        return "-" if x is None else str(x)

    for r in recs:
        tr.write_line(f"{r['what'][:58]:58s} {r['rows']:8d} {f(r['o_max']):>9s} "
                      f"{f(r['o_mean']):>9s} {f(r['floor_max']):>9s} "
                      f"{i(r['o_over_1e-2']):>6s} {i(r['over_1e-2_within_floor']):>8s} "
                      f"{f(r['lse_max']):>9s}")
    path = os.environ.get("RA_PARITY_STATS")
    if path:
        import json
        with open(path, "w") as fh:
            json.dump(recs, fh, indent=1)
