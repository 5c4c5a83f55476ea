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


def row_rel_err(got, ref):
    """max over rows of ||got - ref||_2 / ||ref||_2."""
    got = np.asarray(got, dtype=np.float64).reshape(len(ref), -1)
    ref = np.asarray(ref, dtype=np.float64).reshape(len(ref), -1)
    num = np.linalg.norm(got - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    return float(np.max(num / np.maximum(den, 1e-300)))


def elem_rel_err(got, ref):
    """max |got - ref| / max |ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-300))


# Tolerances (stated for the DASH prefill path: bf16 storage, fp32 accumulation)
HIDDEN_TOL = 2e-2   # hidden states: max row-relative error
DELTA_TOL = 5e-3    # Δ scores: max relative error
CUT_BAND = 1e-3     # selected sets may differ only within this relative band of the cut


@pytest.fixture(scope="session")
def gpu_lib():
    import torch
    from long_context_prefill_tcgen05_b200 import build, dash
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    build.build()
    L = dash.lib()
    assert dash.device_error() == 0
    yield L
    assert dash.device_error() == 0
