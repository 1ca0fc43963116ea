import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _builder():
    """attention_cascade_b200/_build.py loaded by path: importing the package
    itself needs the library that this builds."""
    import importlib.util
    path = os.path.join(ROOT, "attention_cascade_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("attention_cascade_b200_builder", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a); run with -m gpu")
    _builder().build()  # incremental: a no-op when libjev.so is current


@pytest.fixture
def force_tile_rows():
    """Setter of the rows per tensor-core work tile for the test's calls (128:
    the one-Q-tile attention kernel, 256: the two-Q-tile one, 0: the plan
    chooses); the automatic choice is restored afterwards."""
    import attention_cascade_b200 as jev
    yield jev.jev_debug_set_tc_tile_rows
    jev.jev_debug_set_tc_tile_rows(0)


@pytest.fixture(scope="session", autouse=True)
def _build_oracle():
    import oracle
    oracle.build()
