import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _load_build_module():
    path = os.path.join(ROOT, "kv_cache_decode_04_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_gqa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")
    # libgqa.so and libgqa_debug.so are build products (not committed); make sure
    # they match the sources
    _load_build_module().build_all()


def cuda_ok():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="session")
def gqa():
    import kv_cache_decode_04_b200 as m
    return m
