import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: oracle work of more than a few seconds")


def ensure_built():
    """Build libqlora_nf4.so if stale, without importing the package first
    (the package loads the library at import time)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_qnf4_build", os.path.join(ROOT, "bit_nf4_quantized_pack_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def load_golden(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        return json.load(f)


@pytest.fixture
def golden():
    return load_golden
