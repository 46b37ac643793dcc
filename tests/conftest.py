import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def golden():
    return read_golden


@pytest.fixture(params=[1, 2], ids=["cluster", "flat"])
def decode_policy(request):
    """Runs a GPU test once per decode kernel: thread-block clusters, then the
    grid-wide kernel wherever it applies (sizes it does not cover fall back to
    clusters).  The planner's default choice is one of the two."""
    import token_level_sparse_fwht_b200 as ad
    ad.set_decode_policy(request.param)
    yield request.param
    ad.set_decode_policy(0)
