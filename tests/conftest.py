import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def _num(v):
    if isinstance(v, list):
        return [_num(x) for x in v]
    if isinstance(v, str):
        return {"ln3": float(np.float32(np.log(3.0))), "-inf": -np.inf, "inf": np.inf,
                "-0": -0.0}[v]
    return v


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        d = json.load(f)
    return d, _num


@pytest.fixture
def golden():
    return load_golden
