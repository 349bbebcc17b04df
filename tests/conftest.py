import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built liblitela.so")


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()


@pytest.fixture
def paired_min_chunk():
    """Sets the chunk length from which forward calls take the paired fused form (so that small
    shapes, which the oracle finishes quickly, reach it) and restores the default afterwards."""
    import linear_attention_diffusion_litela_b200 as ll
    prev = []

    def set_(tokens):
        prev.append(ll.lite_la_set_paired_min_chunk(tokens))

    yield set_
    if prev:
        ll.lite_la_set_paired_min_chunk(prev[0])
