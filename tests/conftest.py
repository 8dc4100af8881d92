import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def _load_file(name, path):
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) GPU; run with -m gpu")
    # A fresh checkout has no built libraries (they are not committed).
    _load_file("_ag_build", os.path.join(ROOT, "long_context_genomics_b200", "build.py")).ensure_built()
    _load_file("_oracle_build", os.path.join(ROOT, "oracle", "build.py")).ensure_built()


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    return oracle.default()
