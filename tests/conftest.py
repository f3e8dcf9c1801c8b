import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library_if_stale():
    """Compile libdsa_b200.so (nvcc, sm_100a) when it is missing or older than
    its sources and nvcc is present; the package refuses to import without it."""
    import importlib.util
    path = os.path.join(ROOT, "sparse_attention_logits_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("_dsa_b200_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    if not mod.up_to_date():
        try:
            mod.nvcc()
        except RuntimeError:
            return
        mod.build_library()


def pytest_configure(config):
    _build_library_if_stale()
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)
