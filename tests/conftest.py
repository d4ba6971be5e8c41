import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_sessionstart(session):
    """Build libdflash.so before collection unless the library present was
    compiled from exactly these sources (test modules import the package,
    which loads the library on import).  The check compares a hash of the
    sources with the one recorded at build time, so a library left over from
    other sources is rebuilt rather than tested."""
    import importlib.util
    path = os.path.join(ROOT, "block_draft_selection_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_dflash_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


@pytest.fixture(scope="session")
def golden():
    import json

    def load(name):
        with open(os.path.join(GOLDEN, name)) as f:
            return json.load(f)
    return load
