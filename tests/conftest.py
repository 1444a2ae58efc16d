import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a)")
    config.addinivalue_line("markers", "slow: large CPU case")


def read_golden(name: str) -> dict:
    """Parse a ``key = v1 v2 ...`` fixture; '#' lines are comments."""
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, vals = line.partition("=")
            out[key.strip()] = [float(v) for v in vals.split()]
    return out


@pytest.fixture(scope="session")
def golden():
    return read_golden


@pytest.fixture(params=["on", "off", "auto"])
def fusion(request, monkeypatch):
    """Runs a test with the few-token fused linear (the product kernel
    quantising its own input) forced on, off, or chosen by the library
    (BITLINEAR_LINEAR_FUSION, read on every call)."""
    monkeypatch.setenv("BITLINEAR_LINEAR_FUSION", request.param)
    return request.param
