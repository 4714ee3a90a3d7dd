import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libfk.so")
    config.addinivalue_line("markers", "slow: full-size workload case (several seconds or more)")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()


def pytest_terminal_summary(terminalreporter):
    """Print the parity statistics of every label comparison of the run."""
    try:
        from tests.parity import STATS
    except Exception:
        return
    if not STATS:
        return
    tr = terminalreporter
    tr.section("parity statistics (label comparisons against the oracle)")
    keys = ["N", "mismatch", "near_tie_points", "fp32_ties", "centroid_rel_l2", "slack", "empty_clusters",
            "max_log_err", "tol"]
    for d in STATS:
        tr.write_line(d["case"] + ": " + ", ".join(f"{k}={d[k]:.3g}" if isinstance(d.get(k), float)
                                                   else f"{k}={d[k]}" for k in keys if k in d))
