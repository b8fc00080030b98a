import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large host-side inputs")
    # Build the in-tree native libraries (no-op when up to date): the CUDA
    # library cross-compiles without a GPU; the oracle is plain C.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_pa_build", os.path.join(ROOT, "paged_kv_cache_333_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build_all()
    import oracle
    oracle.build()


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "worked_examples.json")) as f:
        return json.load(f)
