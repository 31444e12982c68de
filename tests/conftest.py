import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# the mutation test runs the pins against a copy of the oracle package with a
# planted mistake; ORACLE_PKG names the folder that holds that copy
if os.environ.get("ORACLE_PKG"):
    sys.path.insert(0, os.environ["ORACLE_PKG"])


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
