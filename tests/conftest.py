import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    # test modules import the package (which loads libtbq4.so) at collection
    build_library()


def pytest_collection_modifyitems(config, items):
    # A gpu test on a machine without a device is a hard failure, not a skip,
    # when it is selected explicitly with -m gpu; otherwise it is skipped.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    markexpr = config.getoption("-m") or ""
    if has_gpu or "gpu" in markexpr and "not gpu" not in markexpr:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def build_library():
    """Build libtbq4.so in-tree if it is missing or older than its sources
    (loads build.py by path so the package is imported only afterwards)."""
    import importlib.util
    path = os.path.join(ROOT, "long_context_attention_tbq4_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_tbq4_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
