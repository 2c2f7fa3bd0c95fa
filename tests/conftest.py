import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_lib():
    """The product library, built in-tree if missing; GPU tests only."""
    if not gpu_available():
        pytest.skip("no CUDA device")
    from kv_cache_early_art_b200 import build
    build.build_library()
    import kv_cache_early_art_b200 as art
    return art


@pytest.fixture(autouse=True)
def _poison_shared_memory(request):
    """With ART_POISON_SMEM=nan or =neginf, every GPU test starts with all
    shared memory filled with that pattern, so a kernel that reads shared
    memory it never wrote gives a wrong (non-finite) result instead of
    passing on whatever an earlier kernel left there."""
    mode = os.environ.get("ART_POISON_SMEM", "")
    if mode and request.node.get_closest_marker("gpu") is not None and gpu_available():
        from tests import smem_poison
        smem_poison.poison({"nan": smem_poison.NAN, "neginf": smem_poison.NEG_INF}[mode])
    yield
