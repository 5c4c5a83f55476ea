import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: CPU test taking more than a few seconds")


def to_np(t):
    """Exact widening of a (bf16/fp32) torch tensor to a float64 numpy array."""
    return t.detach().cpu().double().numpy()


def layers_np(layers):
    return [{k: to_np(v) for k, v in w.items()} for w in layers]


@pytest.fixture(scope="session")
def tiny_stack():
    from long_context_prefill_tcgen05_b200 import inputs
    dims = inputs.TINY
    layers = inputs.make_layers(dims, seed=0)
    h0, _ = inputs.make_hidden(512, dims.d_model, seed=0)
    return dims, layers, h0
