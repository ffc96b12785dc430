import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def cuda_lib():
    """The product binding; a GPU test that cannot load it fails, it never falls back."""
    import torch

    if not torch.cuda.is_available():
        pytest.fail("gpu-marked test run without a visible CUDA device")
    import causal_gqa_attention_sm_b200 as nea

    return nea
