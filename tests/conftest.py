import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of host work)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU on this host")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture
def gemm_variant():
    """Selects the bf16 grouped-GEMM kernel for one test (moe_set_gemm_variant)
    and restores the automatic choice afterwards."""
    from routing_grouped_expert_moe_b200 import binding
    chosen = []

    def set_variant(v):
        binding.set_gemm_variant(v)
        chosen.append(v)

    yield set_variant
    if chosen:
        binding.set_gemm_variant(0)
