import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    # The library is a build artefact (not in version control): compile it with nvcc
    # (sm_100a, no GPU needed) when a fresh checkout does not have it yet.
    lib = os.path.join(ROOT, "audio_diffusion_transformer_h3_b200", "libh3attn.so")
    if not os.path.exists(lib):
        import importlib.util
        path = os.path.join(ROOT, "audio_diffusion_transformer_h3_b200", "build.py")
        spec = importlib.util.spec_from_file_location("h3attn_build", path)
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build(force=True)


def _gpu_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _gpu_ok():
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
