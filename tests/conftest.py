import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


@pytest.fixture(scope="session", autouse=True)
def _built_libraries():
    """Build the oracle and the input generator once per session (host compilers only)."""
    import oracle
    from long_context_prefill_trianglemix_b200 import build

    oracle.build()
    build.build_inputs()
    yield
