import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size case, minutes of host time for the oracle")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def schedule_from_golden(entry):
    """(a, b, c) list from a coefficient-table fixture entry."""
    if "steps" in entry:
        return [tuple(float(v) for v in s) for s in entry["steps"]]
    d = float(entry["denominator"])
    return [tuple(v / d for v in s) for s in entry["numerators"]]


@pytest.fixture(scope="session")
def coeff_tables():
    tabs = load_golden("coefficient_tables.json")
    return {k: schedule_from_golden(v) for k, v in tabs.items() if not k.startswith("_")}
