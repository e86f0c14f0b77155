import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build_oracle()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Worst normwise and per-element relative errors of the parity checks."""
    try:
        import helpers
    except ImportError:
        return
    log = helpers.ERR_LOG
    if not log:
        return
    worst_n = max(log, key=lambda e: e[2])
    worst_e = max(log, key=lambda e: e[3])
    tr = terminalreporter
    tr.write_sep("-", "parity error metrics over %d compared tensors" % len(log))
    tr.write_line("worst normwise max|g-o|/max|o|:             %.3e  (%s, shape %s)" % (worst_n[2], worst_n[0], worst_n[1]))
    tr.write_line("worst per-element |g-o|/(|o|+1e-3 max|o|):  %.3e  (%s, shape %s)" % (worst_e[3], worst_e[0], worst_e[1]))
    path = os.environ.get("M3_ERRLOG")
    if path:
        import json
        with open(path, "w") as f:
            json.dump([{"test": t, "shape": list(s), "normwise": n, "per_element": e} for t, s, n, e in log], f)
