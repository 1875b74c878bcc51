import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionstart(session):
    # the CPU suite loads libpkv.so (allocator, ABI checks): build it when it
    # is missing or older than its sources (nvcc cross-compiles without a GPU)
    import importlib.util
    path = os.path.join(ROOT, "paged_kv_cache_365_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("_pkv_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)  # loads the build script without importing the package
    if not mod.up_to_date():
        mod.build()
