"""dash_layer_forward_noalloc: the decoder block for callers that cannot
allocate device memory (no allocator of their own, or a latency-bound loop
where cudaMalloc / cudaFree could synchronise the device).  Its scratch is a
fixed device array inside the library; it must give the same results as
dash_layer_forward with a caller-provided workspace, call after call.

This file is collected last so that, if it fails, a run stopping at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_prefill_tcgen05_b200 import dash, inputs
from conftest import to_np, row_rel_err, HIDDEN_TOL, DELTA_TOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(stack, l, H, pos=None, max_pos=None, halt=None, delta=None, relative=False):
    M = H.shape[0]
    hctx = None
    if halt is not None:
        active, halted, h_full = halt
        hctx = dash.HaltCtx(active.data_ptr(), halted.data_ptr(), h_full.data_ptr(), h_full.shape[0])
        pos = active
    max_pos = (h_full.shape[0] if halt is not None else M) if max_pos is None else max_pos
    return dash.lib().dash_layer_forward_noalloc(
        ctypes.byref(stack.dims), ctypes.pointer(stack.layers[l]), ctypes.c_void_p(H.data_ptr()), M,
        None if pos is None else ctypes.c_void_p(pos.data_ptr()), max_pos,
        ctypes.byref(hctx) if hctx is not None else None,
        None if delta is None else ctypes.c_void_p(delta.data_ptr()), int(relative),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_layer_matches_workspace_layer(gpu_lib, tiny_stack):
    dims, layers, h0 = tiny_stack
    stack = dash.Stack(dims, [{k: v.to(DEV) for k, v in w.items()} for w in layers])
    T = h0.shape[0]
    ref = h0.to(DEV).clone()
    ref_delta = torch.empty(T, device=DEV)
    dash.layer_forward(stack, 1, ref, delta=ref_delta)
    for _ in range(2):  # two calls in a row share the same scratch
        H = h0.to(DEV).clone()
        delta = torch.empty(T, device=DEV)
        assert _noalloc(stack, 1, H, delta=delta) == 0
        assert dash.device_error() == 0
        assert row_rel_err(to_np(H), to_np(ref)) < HIDDEN_TOL
        d, rd = delta.cpu().numpy(), ref_delta.cpu().numpy()
        assert np.max(np.abs(d - rd) / rd) < DELTA_TOL

    # halt-mode context, twice in a row
    rng = np.random.default_rng(3)
    idx = np.sort(rng.choice(T, 150, replace=False))
    halted = np.setdiff1d(np.arange(T), idx)
    ti = torch.tensor(idx, dtype=torch.int32, device=DEV)
    th = torch.tensor(halted, dtype=torch.int32, device=DEV)
    hf = h0.to(DEV)
    ref = hf[ti.long()].contiguous()
    dash.layer_forward(stack, 2, ref, halt=(ti, th, hf))
    for _ in range(2):
        H = hf[ti.long()].contiguous()
        assert _noalloc(stack, 2, H, halt=(ti, th, hf)) == 0
        assert dash.device_error() == 0
        assert row_rel_err(to_np(H), to_np(ref)) < HIDDEN_TOL


def test_noalloc_rejects_shapes_beyond_its_scratch(gpu_lib):
    dims = inputs.QWEN7B
    qd = dash.Dims(dims.n_layers, dims.d_model, dims.n_heads, dims.n_kv_heads, dims.head_dim, dims.ffn_dim,
                   dims.rms_eps, dims.rope_theta)
    fake = dash.LayerWeights(*([1 << 20] * 7))
    # 32768 rows of a 7B-shaped block need gigabytes of scratch: rejected before any launch
    st = dash.lib().dash_layer_forward_noalloc(ctypes.byref(qd), ctypes.byref(fake), ctypes.c_void_p(1 << 20),
                                               32768, None, 32768, None, None, 0, None)
    assert st == 4
