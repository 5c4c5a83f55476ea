"""dash_layer_forward_noalloc: the decoder block for callers that cannot
allocate device memory (no allocator of their own, or a latency-bound loop
where cudaMalloc / cudaFree could synchronise the device).  Its scratch is a
fixed device array inside the library.  It runs the same kernels as
dash_layer_forward with a caller-provided workspace, so the two must agree
bit for bit, call after call -- also when the array still holds a previous
call's data of another shape, so that reading stale scratch would show.

This file is collected last so that, if it fails, a run stopping at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_prefill_tcgen05_b200 import dash, inputs

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


def _scribble(stack, dims, seed):
    """A no-alloc call of another shape, other positions and other data: it
    leaves the shared scratch full of values the next call must not read."""
    T = 300
    h, _ = inputs.make_hidden(T, dims.d_model, seed=seed)
    pos = torch.tensor(np.sort(np.random.default_rng(seed).choice(900, T, replace=False)), dtype=torch.int32,
                       device=DEV)
    H = (h.to(DEV) * 3).contiguous()
    delta = torch.empty(T, device=DEV)
    assert _noalloc(stack, 3, H, pos=pos, max_pos=900, delta=delta, relative=True) == 0
    assert dash.device_error() == 0


def test_noalloc_layer_bitwise_equals_workspace_layer(gpu_lib, tiny_stack):
    dims, layers, h0 = tiny_stack
    stack = dash.Stack(dims, [{k: v.to(DEV) for k, v in w.items()} for w in layers])
    T = h0.shape[0]
    ref = h0.to(DEV).clone()
    ref_delta = torch.empty(T, device=DEV)
    dash.layer_forward(stack, 1, ref, delta=ref_delta)
    for call in range(2):  # two checked calls in a row share the scratch
        _scribble(stack, dims, seed=40 + call)
        H = h0.to(DEV).clone()
        delta = torch.full((T,), float("nan"), device=DEV)
        assert _noalloc(stack, 1, H, delta=delta) == 0
        assert dash.device_error() == 0
        assert torch.equal(H, ref)
        assert torch.equal(delta, ref_delta)

    # halt-mode context (queries at original positions, keys over all rows)
    rng = np.random.default_rng(3)
    idx = np.sort(rng.choice(T, 150, replace=False))
    halted = np.setdiff1d(np.arange(T), idx)
    ti = torch.tensor(idx, dtype=torch.int32, device=DEV)
    th = torch.tensor(halted, dtype=torch.int32, device=DEV)
    hf = h0.to(DEV)
    ref = hf[ti.long()].contiguous()
    ref_delta = torch.empty(len(idx), device=DEV)
    dash.layer_forward(stack, 2, ref, halt=(ti, th, hf), delta=ref_delta)
    for call in range(2):
        _scribble(stack, dims, seed=50 + call)
        H = hf[ti.long()].contiguous()
        delta = torch.full((len(idx),), float("nan"), device=DEV)
        assert _noalloc(stack, 2, H, halt=(ti, th, hf), delta=delta) == 0
        assert dash.device_error() == 0
        assert torch.equal(H, ref)
        assert torch.equal(delta, ref_delta)


def test_noalloc_rejects_shapes_beyond_its_scratch(gpu_lib):
    dims = inputs.QWEN7B
    qd = dash.Dims(dims.n_layers, dims.d_model, dims.n_heads, dims.n_kv_heads, dims.head_dim, dims.ffn_dim,
                   dims.rms_eps, dims.rope_theta)
    fake = dash.LayerWeights(*([1 << 20] * 7))
    # 32768 rows of a 7B-shaped block need gigabytes of scratch: rejected before any launch
    st = dash.lib().dash_layer_forward_noalloc(ctypes.byref(qd), ctypes.byref(fake), ctypes.c_void_p(1 << 20),
                                               32768, None, 32768, None, None, 0, None)
    assert st == 4
