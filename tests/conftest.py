import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on CPU")


@pytest.fixture(scope="session")
def oracle_lib():
    from oracle import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Achieved parity errors (GPU against the oracle), per comparison."""
    mod = sys.modules.get("parity_util")
    log = getattr(mod, "ERROR_LOG", None) if mod else None
    if not log:
        return
    worst = {}
    for r in log:
        w = worst.setdefault(r["case"], dict(r, n=0))
        w["n"] += 1
        for key in ("out_max_abs", "out_rel", "row_rel", "lse_max_abs", "score_rel"):
            if r[key] is not None and (w[key] is None or r[key] > w[key]):
                w[key] = r[key]
        w["out_max_ref"] = max(w["out_max_ref"], r["out_max_ref"])
    tr = terminalreporter
    tr.section("parity errors achieved (worst per case)")
    tr.write_line(f"{'case':70s} {'n':>3s} {'O max abs':>10s} {'max|O_ref|':>10s} {'O rel':>9s} "
                  f"{'row rel':>9s} {'LSE abs':>9s} {'score rel':>9s}")
    fmt = lambda x: f"{x:9.2e}" if x is not None else f"{'-':>9s}"
    for case, w in worst.items():
        tr.write_line(f"{case[-70:]:70s} {w['n']:3d} {w['out_max_abs']:10.3e} {w['out_max_ref']:10.3e} "
                      f"{fmt(w['out_rel'])} {fmt(w['row_rel'])} {fmt(w['lse_max_abs'])} {fmt(w['score_rel'])}")
