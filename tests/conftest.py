import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _load_by_path(name, path):
    import importlib.util
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _build_libraries():
    """Build the oracle and the CUDA library in-tree when missing or stale (nvcc
    cross-compiles for sm_100a without a GPU).  The build scripts are loaded by
    path: importing the packages would load the libraries they build."""
    _load_by_path("_rsq_oracle_build", os.path.join(ROOT, "oracle", "build.py")).build()
    _load_by_path("_rsq_lib_build", os.path.join(ROOT, "ssm_decode_02_b200", "build.py")).build()


def pytest_configure(config):
    _build_libraries()
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU statistical test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
