import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    # temporary files (compiled C probes of the ABI) stay inside the repository
    if not config.option.basetemp:
        config.option.basetemp = os.path.join(ROOT, ".pytest_tmp")
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a)")
    config.addinivalue_line("markers", "slow: large parity case (full-size workload)")


def load_golden(name: str) -> dict:
    """Parse a golden text fixture ("key: v0 v1 ..." lines, '#' comments)."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, vals = line.split(":", 1)
            out[key.strip()] = [float(v) for v in vals.split()]
    return out


@pytest.fixture(scope="session")
def hand_cases():
    return load_golden("hand_cases.txt")
