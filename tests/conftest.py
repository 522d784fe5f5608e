import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large full-size workload")
    # The library is built in-tree (nvcc cross-compiles without a GPU); the build is
    # incremental, so this is a no-op when libftmoe.so is current.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_ftmoe_build", os.path.join(ROOT, "moe_expert_offload_top_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped, not failed, where no device exists; the CPU suite
    # never needs a GPU.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
