"""GPU parity of generation on the DASH KV cache (dash_prefill_kv,
dash_prefill_varlen_kv, dash_decode_attention, dash_decode_step) against the
CPU oracle's return_kv prefill and dash_decode.

The oracle runs free (its own selection); each test first checks that the
GPU chose the same active set, so both sides cache the same rows.
"""
import numpy as np
import pytest
import torch

import oracle as O
from long_context_prefill_tcgen05_b200 import dash, inputs
from conftest import to_np, layers_np, row_rel_err, HIDDEN_TOL

pytestmark = pytest.mark.gpu
DEV = "cuda"
# bf16 keys/values from bf16 layer inputs: one rounding (2^-9 relative) on
# fp32-accumulated projections; rows are compared by relative L2 error.
KV_TOL = 1e-2


def _dev_layers(layers):
    return [{k: v.to(DEV) for k, v in w.items()} for w in layers]


@pytest.fixture(scope="module")
def tiny(gpu_lib, tiny_stack):
    dims, layers, h0 = tiny_stack
    return dims, h0, dash.Stack(dims, _dev_layers(layers)), layers_np(layers)


def _kv_rows(k):
    return np.asarray(k, np.float64).reshape(len(k), -1)


def _check_cache(cache, s, ref_kv, tol_first=KV_TOL, tol=HIDDEN_TOL):
    for l, (rk, rv, rp) in enumerate(ref_kv):
        k, v, p = cache.layer(s, l)
        assert k.shape[0] == len(rk), (l, k.shape[0], len(rk))
        assert np.array_equal(p.cpu().numpy(), rp)
        t = tol_first if l == 0 else tol
        assert row_rel_err(to_np(k), _kv_rows(rk)) < t, l
        assert row_rel_err(to_np(v), _kv_rows(rv)) < t, l


def _new_tokens(n, d, seed):
    return inputs.make_hidden(n, d, seed=seed)[0]


# ------------------------------------------------------ prefill with cache
@pytest.mark.parametrize("mode", ["prune", "halt", "dense"])
def test_prefill_kv_cache_matches_oracle(tiny, mode):
    dims, h0, stack, L = tiny
    T = 512
    cache = dash.KVCache(stack, 1, T + 8)
    H = h0.to(DEV).clone()
    idx = torch.full((T,), -1, dtype=torch.int32, device=DEV)
    cfg = dash.make_config(halt_layer=2, mode=mode, keep=0.5)
    K = dash.prefill_kv(stack, H, cfg, cache, idx_out=idx)
    assert dash.device_error() == 0
    if mode == "dense":
        ref = O.dash_prefill(to_np(h0), L, dims.as_dict(), 3, "prune", keep=1.0, return_kv=True)
    else:
        ref = O.dash_prefill(to_np(h0), L, dims.as_dict(), 2, mode, keep=0.5, return_kv=True)
        assert np.array_equal(idx[:K].cpu().numpy(), ref["idx"])
    late = K if mode == "prune" else T
    assert cache.lens() == [T, T, T, late]
    _check_cache(cache, 0, ref["kv"])
    out = to_np(H[:K]) if mode == "prune" else to_np(H)
    assert row_rel_err(out, ref["hidden"]) < HIDDEN_TOL


# ------------------------------------------------------- decode attention
@pytest.mark.parametrize("hq,hkv,hd", [(4, 2, 64), (28, 4, 128), (32, 8, 128), (16, 1, 64)])
@pytest.mark.parametrize("lens", [[1], [127, 128, 129], [300, 5, 1024, 777]])
def test_decode_attention_matches_oracle(gpu_lib, hq, hkv, hd, lens):
    if len(lens) * hkv > 64:
        pytest.skip("more than 64 (sequence, kv head) segments")
    g = torch.Generator().manual_seed(hq * 1000 + sum(lens))
    n = len(lens)
    Q = (torch.randn(n, hq * hd, generator=g) * 2).to(torch.bfloat16)
    kv = [((torch.randn(m, hkv * hd, generator=g) * 2).to(torch.bfloat16),
           torch.randn(m, hkv * hd, generator=g).to(torch.bfloat16)) for m in lens]
    out = dash.decode_attention(Q.to(DEV), [(k.to(DEV), v.to(DEV)) for k, v in kv], hq, hkv, hd)
    assert dash.device_error() == 0
    for s, m in enumerate(lens):
        k, v = kv[s]
        ref = O.causal_gqa_attention(to_np(Q[s]).reshape(1, hq, hd), to_np(k).reshape(m, hkv, hd),
                                     to_np(v).reshape(m, hkv, hd), [m - 1], np.arange(m))
        got = to_np(out[s].cpu()).reshape(hq, hd)
        assert row_rel_err(got, ref[0]) < 1e-2, s


def test_decode_attention_long_cache_spans_many_ctas(gpu_lib):
    # Qwen-shaped group at 32K + a ragged tail: the key range is split over
    # one wave of CTAs and merged by the combine kernel.
    hq, hkv, hd, m = 28, 4, 128, 32768 + 77
    g = torch.Generator().manual_seed(3)
    Q = (torch.randn(1, hq * hd, generator=g) * 3).to(torch.bfloat16)
    k = (torch.randn(m, hkv * hd, generator=g) * 3).to(torch.bfloat16)
    v = torch.randn(m, hkv * hd, generator=g).to(torch.bfloat16)
    out = dash.decode_attention(Q.to(DEV), [(k.to(DEV), v.to(DEV))], hq, hkv, hd)
    assert dash.device_error() == 0
    ref = O.causal_gqa_attention(to_np(Q).reshape(1, hq, hd), to_np(k).reshape(m, hkv, hd),
                                 to_np(v).reshape(m, hkv, hd), [m - 1], np.arange(m))
    assert row_rel_err(to_np(out.cpu()).reshape(hq, hd), ref[0]) < 1e-2


# --------------------------------------------------------- decode steps
@pytest.mark.parametrize("mode", ["prune", "halt", "dense"])
def test_decode_steps_tiny_match_oracle(tiny, mode):
    dims, h0, stack, L = tiny
    T, steps = 300, 3
    cache = dash.KVCache(stack, 1, T + steps)
    H = h0[:T].to(DEV).clone()
    cfg = dash.make_config(halt_layer=1, mode=mode, keep=0.4)
    idx = torch.full((T,), -1, dtype=torch.int32, device=DEV)
    K = dash.prefill_kv(stack, H, cfg, cache, idx_out=idx)
    if mode == "dense":
        ref = O.dash_prefill(to_np(h0[:T]), L, dims.as_dict(), 3, "prune", keep=1.0, return_kv=True)
    else:
        ref = O.dash_prefill(to_np(h0[:T]), L, dims.as_dict(), 1, mode, keep=0.4, return_kv=True)
        assert np.array_equal(idx[:K].cpu().numpy(), ref["idx"])
    kv = ref["kv"]
    x = _new_tokens(steps, dims.d_model, seed=11)
    for t in range(steps):
        X = x[t:t + 1].to(DEV).clone()
        dash.decode_step(stack, X, [T + t], cache)
        assert dash.device_error() == 0
        y, kv = O.dash_decode(to_np(x[t:t + 1]), [T + t], kv, L, dims.as_dict())
        assert row_rel_err(to_np(X), y) < HIDDEN_TOL, t
    late = (K if mode == "prune" else T) + steps
    assert cache.lens() == [T + steps, T + steps, late, late]
    _check_cache(cache, 0, kv)


def test_decode_on_empty_cache_attends_to_itself(tiny):
    dims, h0, stack, L = tiny
    cache = dash.KVCache(stack, 1, 4)
    x = _new_tokens(2, dims.d_model, seed=12)
    X = x.to(DEV).clone()[:1]
    dash.decode_step(stack, X, [0], cache)
    empty = [(np.zeros((0, dims.n_kv_heads, dims.head_dim)),) * 2 + (np.zeros(0, np.int64),)] * len(L)
    y, kv = O.dash_decode(to_np(x[:1]), [0], empty, L, dims.as_dict())
    assert row_rel_err(to_np(X), y) < HIDDEN_TOL
    X2 = x.to(DEV).clone()[1:]
    dash.decode_step(stack, X2, [1], cache)
    y2, _ = O.dash_decode(to_np(x[1:]), [1], kv, L, dims.as_dict())
    assert row_rel_err(to_np(X2), y2) < HIDDEN_TOL
    assert cache.lens() == [2] * len(L)


@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_decode_batch_after_varlen_prefill(tiny, mode):
    # three sequences of different lengths prefilled together, then one
    # generation step for all three in one call
    dims, h0, stack, L = tiny
    cu = [0, 200, 329, 512]
    nseq = 3
    cache = dash.KVCache(stack, nseq, 260)
    H = h0.to(DEV).clone()
    cfg = dash.make_config(halt_layer=2, mode=mode, keep=0.5)
    idx = torch.full((512,), -1, dtype=torch.int32, device=DEV)
    K, counts = dash.prefill_varlen_kv(stack, H, cu, cfg, cache, idx_out=idx)
    assert dash.device_error() == 0
    ref = O.dash_prefill_varlen(to_np(h0), cu, L, dims.as_dict(), 2, mode, keep=0.5, return_kv=True)
    assert np.array_equal(idx[:K].cpu().numpy(), ref["idx"])
    for s in range(nseq):
        _check_cache(cache, s, ref["kv"][s])
    x = _new_tokens(nseq, dims.d_model, seed=13)
    X = x.to(DEV).clone()
    lens = [cu[s + 1] - cu[s] for s in range(nseq)]
    dash.decode_step(stack, X, lens, cache)
    assert dash.device_error() == 0
    for s in range(nseq):
        y, kv = O.dash_decode(to_np(x[s:s + 1]), [lens[s]], ref["kv"][s], L, dims.as_dict())
        assert row_rel_err(to_np(X[s:s + 1]), y) < HIDDEN_TOL, s
        _check_cache(cache, s, kv)


# ----------------------------------------------------- Qwen-shaped layer
@pytest.mark.parametrize("T", [32768, 16384 + 37])
def test_decode_qwen_layer_full_size(gpu_lib, T):
    # One Qwen2.5-7B-shaped layer: the prefill caches all T rows (the sizes
    # of a dense and a pruned layer at 32K), then one token is generated.
    # Layer 0 sees the seeded input directly, so the oracle runs free.
    dims = inputs.QWEN7B
    layers = inputs.make_layers(dims, seed=0, n_layers=1)
    stack = dash.Stack(dims, _dev_layers(layers))
    h0 = inputs.make_hidden(T, dims.d_model, seed=0)[0]
    cache = dash.KVCache(stack, 1, T + 1)
    H = h0.to(DEV).clone()
    dash.prefill_kv(stack, H, dash.make_config(mode="dense"), cache)
    x = _new_tokens(1, dims.d_model, seed=21)
    X = x.to(DEV).clone()
    dash.decode_step(stack, X, [T], cache)
    assert dash.device_error() == 0
    Ln = layers_np(layers)
    k, v = O.layer_kv(to_np(h0), np.arange(T), Ln[0], dims.as_dict())
    y, kv = O.dash_decode(to_np(x), [T], [(k, v, np.arange(T))], Ln, dims.as_dict())
    assert row_rel_err(to_np(X), y) < HIDDEN_TOL
    ck, cv, cp = cache.layer(0, 0)
    assert ck.shape[0] == T + 1 and int(cp[-1]) == T
    rows = np.r_[np.arange(0, T, 997), T]
    assert row_rel_err(to_np(ck[rows].cpu()), _kv_rows(kv[0][0][rows])) < KV_TOL
    assert row_rel_err(to_np(cv[rows].cpu()), _kv_rows(kv[0][1][rows])) < KV_TOL


@pytest.mark.parametrize("tensor_cores", [True, False])
@pytest.mark.parametrize("nseq", [3, 5, 8])
def test_decode_qwen_layer_many_sequences(gpu_lib, nseq, tensor_cores):
    # One Qwen2.5-7B-shaped layer, nseq sequences with short caches of seeded
    # random rows, in both forms of the projections: on the tensor cores
    # (K split over the SMs for QKV, o_proj and down) and as CUDA-core GEMVs
    # (where down's input rows, nseq x 18944 values, exceed what the GEMV
    # stages in shared memory beyond 4 sequences, so it runs in groups of 4).
    prev = dash.set_decode_tensor_cores(tensor_cores)
    try:
        _many_sequences_case(nseq)
    finally:
        dash.set_decode_tensor_cores(prev)


def _many_sequences_case(nseq):
    dims = inputs.QWEN7B
    layers = inputs.make_layers(dims, seed=3, n_layers=1)
    stack = dash.Stack(dims, _dev_layers(layers))
    lens = [37, 300, 129, 1, 200, 64, 255, 90][:nseq]
    cache = dash.KVCache(stack, nseq, max(lens) + 1)
    hkv, hd = dims.n_kv_heads, dims.head_dim
    g = torch.Generator().manual_seed(5)
    ref_kv = []
    for s, n in enumerate(lens):
        k = torch.randn(n, hkv * hd, generator=g).to(torch.bfloat16)
        v = torch.randn(n, hkv * hd, generator=g).to(torch.bfloat16)
        cache.k[s][:n] = k.to(DEV)
        cache.v[s][:n] = v.to(DEV)
        cache.pos[s][:n] = torch.arange(n, dtype=torch.int32, device=DEV)
        cache.desc[s].len = n
        ref_kv.append((to_np(k).reshape(n, hkv, hd), to_np(v).reshape(n, hkv, hd), np.arange(n)))
    x = _new_tokens(nseq, dims.d_model, seed=23)
    X = x.to(DEV).clone()
    dash.decode_step(stack, X, lens, cache)
    assert dash.device_error() == 0
    Ln = layers_np(layers)
    for s, n in enumerate(lens):
        y, kv = O.dash_decode(to_np(x[s:s + 1]), [n], [ref_kv[s]], Ln, dims.as_dict())
        assert row_rel_err(to_np(X[s:s + 1].cpu()), y) < HIDDEN_TOL, s
        ck, cv, cp = cache.layer(s, 0)
        assert ck.shape[0] == n + 1 and int(cp[-1]) == n
        assert row_rel_err(to_np(ck[-1:].cpu()), _kv_rows(kv[0][0][-1:])) < KV_TOL, s


def test_decode_wide_ffn_more_items_than_sms(gpu_lib):
    # A narrow model with a wide FFN (38400 = 300 row blocks of 128): the
    # tensor-core gate/up projection has more items than the device has SMs,
    # so CTAs take a second item (accumulator and weight-ring reuse).
    dims = inputs.ModelDims(2, 256, 4, 2, 64, 38400, 1e4)
    layers = inputs.make_layers(dims, seed=8, n_layers=2)
    stack = dash.Stack(dims, _dev_layers(layers))
    nseq, n = 4, 50
    cache = dash.KVCache(stack, nseq, n + 1)
    kvd = dims.n_kv_heads * dims.head_dim
    g = torch.Generator().manual_seed(9)
    ref_kv = []
    for s in range(nseq):
        per_layer = []
        for l in range(dims.n_layers):
            k = torch.randn(n, kvd, generator=g).to(torch.bfloat16)
            v = torch.randn(n, kvd, generator=g).to(torch.bfloat16)
            i = s * dims.n_layers + l
            cache.k[i][:n] = k.to(DEV)
            cache.v[i][:n] = v.to(DEV)
            cache.pos[i][:n] = torch.arange(n, dtype=torch.int32, device=DEV)
            cache.desc[i].len = n
            per_layer.append((to_np(k).reshape(n, dims.n_kv_heads, dims.head_dim),
                              to_np(v).reshape(n, dims.n_kv_heads, dims.head_dim), np.arange(n)))
        ref_kv.append(per_layer)
    x = _new_tokens(nseq, dims.d_model, seed=24)
    X = x.to(DEV).clone()
    dash.decode_step(stack, X, [n] * nseq, cache)
    assert dash.device_error() == 0
    Ln = layers_np(layers)
    for s in range(nseq):
        y, _ = O.dash_decode(to_np(x[s:s + 1]), [n], ref_kv[s], Ln, dims.as_dict())
        assert row_rel_err(to_np(X[s:s + 1].cpu()), y) < HIDDEN_TOL, s
