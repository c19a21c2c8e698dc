import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    under_test = os.environ.get("PA_ORACLE_UNDER_TEST")
    if under_test:
        # a copy of the oracle package with a planted mistake
        # (tests/test_oracle_mutants.py), loaded under its own name
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "oracle_under_test", os.path.join(under_test, "__init__.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    else:
        import oracle as mod
    mod.build()
    return mod
