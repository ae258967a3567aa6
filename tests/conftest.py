import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Parity records of the full-size workload tests (near-tie counts, largest
# errors against the oracle), printed at the end of the session and, when
# LSH_PARITY_JSON names a file, written there as JSON.
PARITY_RECORDS = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    from oracle import oracle as o
    o.build()
    return o


@pytest.fixture(scope="session")
def parity_record():
    return PARITY_RECORDS


def pytest_terminal_summary(terminalreporter):
    if not PARITY_RECORDS:
        return
    terminalreporter.write_line("parity records (GPU against the fp64 oracle):")
    for rec in PARITY_RECORDS:
        terminalreporter.write_line("PARITY " + json.dumps(rec, sort_keys=True))
    path = os.environ.get("LSH_PARITY_JSON")
    if path:
        with open(path, "w") as f:
            json.dump(PARITY_RECORDS, f, indent=1, sort_keys=True)
