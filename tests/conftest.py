import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs an NVIDIA B200 (sm_100a) and the built libgdn.so")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def record_parity(what, err, tau):
    """Appends one measured error ratio max|x - x_ref| / max|x_ref| (and its bar) to
    the JSON-lines file named by GDN_PARITY_LOG, when that variable is set: the
    record of the errors the GPU parity tests measured."""
    path = os.environ.get("GDN_PARITY_LOG")
    if not path:
        return
    import json
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, "what": what, "err": err, "tau": tau}) + "\n")
