"""GPU parity of dash_layer_forward and dash_prefill against the CPU oracle.

Tiny stack (4 layers, d=256, T=512): full end-to-end comparison with the
free-running oracle (the active sets must come out identical).  Qwen2.5-7B-
shaped stack: one layer at a time on seeded layer inputs, checked on sampled
query rows at the full T=32768 launch shapes the benchmark times, plus
properties that hold at any size.  Selection is also checked as the oracle's
rule applied to the GPU's own fp32 Δ: an integer decision taken from floating
point is compared in the kernel's precision.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from long_context_prefill_tcgen05_b200 import dash, inputs
from conftest import to_np, layers_np, row_rel_err, HIDDEN_TOL, DELTA_TOL, CUT_BAND

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev_layers(layers):
    return [{k: v.to(DEV) for k, v in w.items()} for w in layers]


@pytest.fixture(scope="module")
def tiny(gpu_lib, tiny_stack):
    dims, layers, h0 = tiny_stack
    return dims, h0, dash.Stack(dims, _dev_layers(layers)), layers_np(layers)


def _prefill(stack, h0, **kw):
    H = h0.to(DEV).clone()
    T = H.shape[0]
    idx = torch.full((T,), -1, dtype=torch.int32, device=DEV)
    delta = torch.empty(T, dtype=torch.float32, device=DEV)
    K = dash.prefill(stack, H, dash.make_config(**kw), idx_out=idx, delta_out=delta)
    assert dash.device_error() == 0
    return H.cpu(), idx[:K].cpu().numpy(), delta.cpu().numpy(), K


def _rel(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - b) / np.abs(b)))


def _check_sets(idx, ref_idx, ref_delta, cut):
    diff = np.setxor1d(idx, ref_idx)
    for t in diff:
        assert abs(ref_delta[t] - cut) <= CUT_BAND * abs(cut), (t, ref_delta[t], cut)


def _clear_threshold(delta, q, window=20):
    """A threshold near the q-quantile of the oracle's Δ placed at the middle of
    the widest relative gap between neighbouring values, so no token sits at
    the cut and both sides select the same set (chosen from the oracle only)."""
    d = np.sort(np.asarray(delta, np.float64))
    k = int(q * (len(d) - 1))
    lo, hi = max(0, k - window), min(len(d) - 2, k + window)
    i = max(range(lo, hi + 1), key=lambda j: (d[j + 1] - d[j]) / max(abs(d[j + 1]), 1e-30))
    return float(np.float32(0.5 * (d[i] + d[i + 1])))


def _topk_cut(delta, keep, nf=0, nl=0):
    T = len(delta)
    mid = np.flatnonzero(~O.forced_mask(T, nf, nl))
    k = math.floor(keep * len(mid))
    return np.sort(delta[mid])[::-1][k - 1] if k > 0 else np.inf


# ------------------------------------------------------------- tiny layer
def test_layer_dense_matches_oracle(tiny):
    dims, h0, stack, L = tiny
    T = h0.shape[0]
    H = h0.to(DEV).clone()
    delta = torch.empty(T, device=DEV)
    dash.layer_forward(stack, 0, H, delta=delta)
    pos = np.arange(T)
    ref, u = O.decoder_block(to_np(h0), pos, to_np(h0), pos, L[0], dims.as_dict())
    assert row_rel_err(to_np(H), ref) < HIDDEN_TOL
    assert _rel(delta.cpu().numpy(), O.delta_scores(u)) < DELTA_TOL
    delta_r = torch.empty(T, device=DEV)
    dash.layer_forward(stack, 0, h0.to(DEV).clone(), delta=delta_r, relative=True)
    assert _rel(delta_r.cpu().numpy(), O.delta_scores(u, to_np(h0), True)) < DELTA_TOL


def test_layer_compacted_rows_at_original_positions(tiny):
    dims, h0, stack, L = tiny
    rng = np.random.default_rng(5)
    idx = np.sort(rng.choice(512, 200, replace=False))
    H = h0[idx].to(DEV).contiguous()
    dash.layer_forward(stack, 1, H, pos=torch.tensor(idx, dtype=torch.int32, device=DEV), max_pos=512)
    hn = to_np(h0)[idx]
    ref, _ = O.decoder_block(hn, idx, hn, idx, L[1], dims.as_dict())
    assert row_rel_err(to_np(H), ref) < HIDDEN_TOL


def test_layer_halt_context(tiny):
    dims, h0, stack, L = tiny
    rng = np.random.default_rng(6)
    idx = np.sort(rng.choice(512, 130, replace=False))
    halted = np.setdiff1d(np.arange(512), idx)
    H = h0[idx].to(DEV).contiguous()
    hf = h0.to(DEV)
    ti = torch.tensor(idx, dtype=torch.int32, device=DEV)
    th = torch.tensor(halted, dtype=torch.int32, device=DEV)
    delta = torch.empty(len(idx), device=DEV)
    dash.layer_forward(stack, 3, H, halt=(ti, th, hf), delta=delta)
    ref, u = O.decoder_block(to_np(h0)[idx], idx, to_np(h0), np.arange(512), L[3], dims.as_dict())
    assert row_rel_err(to_np(H), ref) < HIDDEN_TOL
    assert _rel(delta.cpu().numpy(), O.delta_scores(u)) < DELTA_TOL


def test_layer_halt_context_bad_active_index_is_flagged(tiny):
    """An active index past the sequence would address the RoPE table and the
    k / v rows out of range: the QKV epilogue leaves that row unwritten and
    reports INDEX; the context stays usable."""
    dims, h0, stack, L = tiny
    T = 512
    idx = np.arange(0, T, 4)
    halted = np.setdiff1d(np.arange(T), idx)
    bad = idx.copy()
    bad[-1] = T + 5  # ascending, but out of range
    ti = torch.tensor(bad, dtype=torch.int32, device=DEV)
    th = torch.tensor(halted, dtype=torch.int32, device=DEV)
    hf = h0.to(DEV)
    H = hf[torch.tensor(idx, device=DEV).long()].contiguous()
    dash.layer_forward(stack, 3, H, halt=(ti, th, hf))
    assert dash.device_error() == 7  # reported and cleared
    good = torch.tensor(idx, dtype=torch.int32, device=DEV)
    H = hf[good.long()].contiguous()
    dash.layer_forward(stack, 3, H, halt=(good, th, hf))
    assert dash.device_error() == 0
    ref, _ = O.decoder_block(to_np(h0)[idx], idx, to_np(h0), np.arange(T), L[3], dims.as_dict())
    assert row_rel_err(to_np(H), ref) < HIDDEN_TOL


# ----------------------------------------------------------- tiny prefill
@pytest.mark.parametrize("mode", ["prune", "halt"])
@pytest.mark.parametrize("keep,nf,nl", [(0.5, 0, 0), (0.3, 64, 32)])
def test_prefill_tiny_matches_oracle(tiny, mode, keep, nf, nl):
    dims, h0, stack, L = tiny
    Hg, idx, delta, K = _prefill(stack, h0, halt_layer=2, mode=mode, keep=keep, keep_first=nf, keep_last=nl)
    free = O.dash_prefill(to_np(h0), L, dims.as_dict(), 2, mode, keep=keep, keep_first=nf, keep_last=nl)
    assert K == O.topk_count(512, keep, nf, nl) == len(free["idx"])
    assert _rel(delta, free["delta"]) < DELTA_TOL
    assert np.all(np.diff(idx) > 0)
    # the GPU's selection on its own fp32 scores is exactly the oracle's rule
    assert np.array_equal(idx, O.select_topk(delta.astype(np.float64), keep, nf, nl))
    _check_sets(idx, free["idx"], free["delta"], _topk_cut(free["delta"], keep, nf, nl))
    assert np.array_equal(idx, free["idx"])  # no near-tie at the cut on this input: same rows cached
    got = to_np(Hg[:K]) if mode == "prune" else to_np(Hg)
    assert row_rel_err(got, free["hidden"]) < HIDDEN_TOL


def test_prefill_tiny_threshold_relative(tiny):
    dims, h0, stack, L = tiny
    free0 = O.dash_prefill(to_np(h0), L, dims.as_dict(), 1, "halt", keep=1.0, relative=True)
    thr = _clear_threshold(free0["delta"], 0.7)
    Hg, idx, delta, K = _prefill(stack, h0, halt_layer=1, mode="halt", select="threshold", threshold=thr,
                                 relative=True)
    free = O.dash_prefill(to_np(h0), L, dims.as_dict(), 1, "halt", select="threshold", threshold=thr,
                          relative=True)
    assert _rel(delta, free["delta"]) < DELTA_TOL
    assert np.array_equal(idx, O.select_threshold(delta.astype(np.float64), np.float32(thr)))
    _check_sets(idx, free["idx"], free["delta"], thr)
    assert np.array_equal(idx, free["idx"])
    assert row_rel_err(to_np(Hg), free["hidden"]) < HIDDEN_TOL


def test_prefill_tiny_dense_matches_oracle(tiny):
    dims, h0, stack, L = tiny
    Hg, _, _, K = _prefill(stack, h0, mode="dense")
    assert K == 512
    assert row_rel_err(to_np(Hg), O.dense_forward(to_np(h0), L, dims.as_dict())) < HIDDEN_TOL


def test_keep_one_prune_is_bitwise_dense(tiny):
    dims, h0, stack, L = tiny
    Hd, _, _, _ = _prefill(stack, h0, mode="dense")
    Hp, idx, _, K = _prefill(stack, h0, halt_layer=1, mode="prune", keep=1.0)
    Hh, _, _, _ = _prefill(stack, h0, halt_layer=2, mode="halt", keep=1.0)
    assert K == 512 and np.array_equal(idx, np.arange(512))
    assert torch.equal(Hp, Hd) and torch.equal(Hh, Hd)


def test_halted_rows_frozen_at_halting_layer_output(tiny):
    dims, h0, stack, L = tiny
    Hh, idx, _, K = _prefill(stack, h0, halt_layer=1, mode="halt", keep=0.25)
    first2 = dash.Stack(dims, _tiny_layers(dims)[:2])
    Hs, _, _, _ = _prefill(first2, h0, mode="dense")
    halted = np.setdiff1d(np.arange(512), idx)
    assert torch.equal(Hh[halted], Hs[halted])


def _tiny_layers(dims):
    return _dev_layers(inputs.make_layers(dims, seed=0))


def test_prefill_zero_keep(tiny):
    dims, h0, stack, L = tiny
    Hp, idx, _, K = _prefill(stack, h0, halt_layer=2, mode="prune", keep=0.0)
    assert K == 0
    Hh, idx, _, K = _prefill(stack, h0, halt_layer=2, mode="halt", keep=0.0)
    first3 = dash.Stack(dims, _tiny_layers(dims)[:3])
    Hs, _, _, _ = _prefill(first3, h0, mode="dense")
    assert torch.equal(Hh, Hs)


def test_prefill_reports_nonfinite(tiny):
    dims, h0, stack, L = tiny
    bad = h0.clone()
    bad[7, :] = 0  # ||H_7|| = 0 at layer 0 in relative mode -> Δ is not finite
    with pytest.raises(dash.DashError) as e:
        _prefill(stack, bad, halt_layer=0, mode="prune", keep=0.5, relative=True)
    assert e.value.status == 3
    assert dash.device_error() == 3


# ------------------------------------------------- Qwen2.5-7B-shaped layers
@pytest.fixture(scope="module")
def qwen_layer(gpu_lib):
    dims = inputs.QWEN7B
    layers = inputs.make_layers(dims, seed=11, device=DEV, n_layers=1)
    return dims, dash.Stack(dims, layers), {k: to_np(v) for k, v in layers[0].items()}


def _sampled_check(dims, W, h_in, h_out, rows, q_pos, kv_rows, kv_pos, delta=None):
    """Oracle block for the sampled query rows (keys/values from every kv row)."""
    hin = to_np(h_in)
    ref, u = O.decoder_block(hin[rows], q_pos, to_np(kv_rows), kv_pos, W, dims.as_dict())
    assert row_rel_err(to_np(h_out)[rows], ref) < HIDDEN_TOL
    if delta is not None:
        assert _rel(delta[rows], O.delta_scores(u)) < DELTA_TOL


@pytest.mark.slow
def test_qwen_layer_full_T_sampled_rows(qwen_layer):
    dims, stack, W = qwen_layer
    T = 32768
    h0, _ = inputs.make_hidden(T, dims.d_model, seed=21, device=DEV)
    H = h0.clone()
    delta = torch.empty(T, device=DEV)
    dash.layer_forward(stack, 0, H, delta=delta)
    assert dash.device_error() == 0
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 4095, T - 1],
                                     np.random.default_rng(0).choice(T, 250, replace=False)]))
    _sampled_check(dims, W, h0.cpu(), H.cpu(), rows, rows, h0.cpu(), np.arange(T), delta.cpu().numpy())


@pytest.mark.slow
def test_qwen_layer_compacted_prune_shape(qwen_layer):
    dims, stack, W = qwen_layer
    T, K = 32768, 16384
    rng = np.random.default_rng(1)
    idx = np.sort(rng.choice(T, K, replace=False))
    h0, _ = inputs.make_hidden(K, dims.d_model, seed=22, device=DEV)
    H = h0.clone()
    dash.layer_forward(stack, 0, H, pos=torch.tensor(idx, dtype=torch.int32, device=DEV), max_pos=T)
    assert dash.device_error() == 0
    rows = np.sort(rng.choice(K, 256, replace=False))
    _sampled_check(dims, W, h0.cpu(), H.cpu(), rows, idx[rows], h0.cpu(), idx)


@pytest.mark.slow
def test_qwen_layer_halt_shape(qwen_layer):
    dims, stack, W = qwen_layer
    T, K = 32768, 16384
    rng = np.random.default_rng(2)
    idx = np.sort(rng.choice(T, K, replace=False))
    halted = np.setdiff1d(np.arange(T), idx)
    hfull, _ = inputs.make_hidden(T, dims.d_model, seed=23, device=DEV)
    H = hfull[torch.tensor(idx, device=DEV)].contiguous()
    h_in = H.clone()
    ti = torch.tensor(idx, dtype=torch.int32, device=DEV)
    dash.layer_forward(stack, 0, H, halt=(ti, torch.tensor(halted, dtype=torch.int32, device=DEV), hfull))
    assert dash.device_error() == 0
    rows = np.sort(rng.choice(K, 256, replace=False))
    _sampled_check(dims, W, h_in.cpu(), H.cpu(), rows, idx[rows], hfull.cpu(), np.arange(T))


@pytest.mark.parametrize("mode", ["dense", "halt"])
def test_qwen_layer_pair_tiles_match_single_sm_tiles(qwen_layer, mode):
    """Every fused GEMM epilogue (RoPE/QKV split, halted K/V at original rows,
    residual + Δ partial sums, SwiGLU, residual) on SM-pair tiles against the
    single-SM kernel at Qwen2.5-7B widths, ragged row count."""
    dims, stack, W = qwen_layer
    T, K = 4096, 1500
    hfull, _ = inputs.make_hidden(T, dims.d_model, seed=24, device=DEV)
    rng = np.random.default_rng(3)
    idx = np.sort(rng.choice(T, K, replace=False))
    halted = np.setdiff1d(np.arange(T), idx)
    ti = torch.tensor(idx, dtype=torch.int32, device=DEV)
    th = torch.tensor(halted, dtype=torch.int32, device=DEV)

    def run(pairs):
        prev = dash.set_gemm_pairs(pairs)
        try:
            if mode == "dense":
                H = hfull.clone()
                delta = torch.empty(T, device=DEV)
                dash.layer_forward(stack, 0, H, delta=delta)
            else:
                H = hfull[ti.long()].contiguous()
                delta = torch.empty(K, device=DEV)
                dash.layer_forward(stack, 0, H, halt=(ti, th, hfull), delta=delta)
        finally:
            dash.set_gemm_pairs(prev)
        assert dash.device_error() == 0
        return to_np(H.cpu()), delta.cpu().numpy()

    Hp, dp = run(True)
    Hs, ds = run(False)
    assert row_rel_err(Hp, Hs.astype(np.float64)) < 1e-3
    assert _rel(dp, ds.astype(np.float64)) < 1e-4
    rows = np.sort(np.concatenate([[0, len(dp) - 1], rng.choice(len(dp), 14, replace=False)]))
    if mode == "dense":
        _sampled_check(dims, W, hfull.cpu(), torch.from_numpy(Hp), rows, rows, hfull.cpu(), np.arange(T), dp)
    else:
        _sampled_check(dims, W, hfull[ti.long()].cpu(), torch.from_numpy(Hp), rows, idx[rows], hfull.cpu(),
                       np.arange(T), dp)


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_qwen_layer_last_wave_rectangle(qwen_layer, mode):
    """9700 rows at Qwen2.5-7B widths: the QKV GEMM's 684 pair tiles leave a
    last wave of 18, which runs as a rectangle of single-SM tiles (rows 8192
    onwards, the last 768 qkv columns: k and v heads) -- with positions
    (prune) and with the k/v row map of halt mode.  Bitwise equal to the
    all-single-SM layer; sampled rows, including rows of the rectangle,
    against the oracle."""
    dims, stack, W = qwen_layer
    T, M = 16384, 9700
    rng = np.random.default_rng(7)
    idx = np.sort(rng.choice(T, M, replace=False))
    halted = np.setdiff1d(np.arange(T), idx)
    hfull, _ = inputs.make_hidden(T, dims.d_model, seed=25, device=DEV)
    ti = torch.tensor(idx, dtype=torch.int32, device=DEV)
    th = torch.tensor(halted, dtype=torch.int32, device=DEV)

    def run(pairs):
        prev = dash.set_gemm_pairs(pairs)
        try:
            H = hfull[ti.long()].contiguous()
            if mode == "prune":
                dash.layer_forward(stack, 0, H, pos=ti, max_pos=T)
            else:
                dash.layer_forward(stack, 0, H, halt=(ti, th, hfull))
        finally:
            dash.set_gemm_pairs(prev)
        assert dash.device_error() == 0
        return H.cpu()

    Hp, Hs = run(True), run(False)
    assert torch.equal(Hp, Hs)
    rows = np.unique(np.r_[0, M - 1, rng.choice(np.arange(8192, M), 40, replace=False),
                           rng.choice(8192, 24, replace=False)])
    h_in = hfull[ti.long()].cpu()
    if mode == "prune":
        _sampled_check(dims, W, h_in, Hp, rows, idx[rows], h_in, idx)
    else:
        _sampled_check(dims, W, h_in, Hp, rows, idx[rows], hfull.cpu(), np.arange(T))


# ------------------------------------- reduced Qwen-shaped, end to end
def _clear_keep(delta, q, window=400):
    """A keep fraction near q whose top-k cut falls in the widest relative gap
    between neighbouring oracle Δ values within the window (chosen from the
    oracle alone), so the GPU's fp32 Δ cannot reorder rows across the cut."""
    d = np.sort(np.asarray(delta, np.float64))[::-1]
    k0 = int(q * len(d))
    best = max(range(max(1, k0 - window), min(len(d) - 1, k0 + window)),
               key=lambda k: (d[k - 1] - d[k]) / d[k - 1])
    return (best + 0.5) / len(d)  # floor(keep * T) = best


@pytest.fixture(scope="module")
def qwen_reduced(gpu_lib):
    """Qwen2.5-7B widths, 4 layers, T = 2048: halting at layer 1 gives two full
    layers and two on the active set."""
    dims = inputs.QWEN7B
    layers = inputs.make_layers(dims, seed=31, n_layers=4)
    h0, _ = inputs.make_hidden(2048, dims.d_model, seed=32)
    L = layers_np(layers)
    # Δ depends on layers 0..1 only
    d0 = O.dash_prefill(to_np(h0), L[:2], dims.as_dict(), 1, "prune", keep=1.0)["delta"]
    return dims, h0, dash.Stack(dims, _dev_layers(layers)), L, _clear_keep(d0, 0.5)


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_qwen_reduced_prefill_matches_free_oracle(qwen_reduced, mode):
    dims, h0, stack, L, keep = qwen_reduced
    T = h0.shape[0]
    Hg, idx, delta, K = _prefill(stack, h0, halt_layer=1, mode=mode, keep=keep)
    free = O.dash_prefill(to_np(h0), L, dims.as_dict(), 1, mode, keep=keep)
    assert K == O.topk_count(T, keep) == len(free["idx"])
    # Δ at layer 1 sees layer 0's output through the bf16 residual stream
    # (up to 2^-8 relative per element, which the fp64 oracle does not round):
    # 5e-3 holds for 99 % of the tokens, twice that for the worst one.  This
    # is the bf16 path's documented departure from the stated 5e-3; the fp16
    # format holds it on the same case (test_fp16_reduced_prefill_matches_free_oracle),
    # and the per-layer 5e-3 bound is checked teacher-forced in test_qwen_layer_*.
    rel = np.abs(delta.astype(np.float64) - free["delta"]) / free["delta"]
    assert np.quantile(rel, 0.99) < DELTA_TOL
    assert rel.max() < 2 * DELTA_TOL
    assert np.array_equal(idx, O.select_topk(delta.astype(np.float64), keep))
    _check_sets(idx, free["idx"], free["delta"], _topk_cut(free["delta"], keep))
    # Rows may swap across the cut only within the band _check_sets allows;
    # compare the rows both kept (prune) or that both treated alike (halt).
    # One swapped key moves the others' attention by ~1/K of its mass, far
    # inside the hidden-state tolerance.
    common = np.intersect1d(idx, free["idx"])
    if mode == "prune":
        got = to_np(Hg[:K])[np.searchsorted(idx, common)]
        ref = free["hidden"][np.searchsorted(free["idx"], common)]
    else:
        same = np.setdiff1d(np.arange(T), np.setxor1d(idx, free["idx"]))
        got, ref = to_np(Hg)[same], free["hidden"][same]
    assert len(common) >= K - 4
    assert row_rel_err(got, ref) < HIDDEN_TOL


# ----------------------------------------- full-size prefill properties
@pytest.mark.slow
@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_qwen_prefill_32k_properties(gpu_lib, mode):
    """The benchmark's workload (28 layers, T=32768, halt at 11, keep 0.5):
    count, order, selection = the oracle rule on the GPU's own Δ, finite output."""
    dims = inputs.QWEN7B
    stack = dash.Stack(dims, inputs.make_layers(dims, seed=0, device=DEV))
    h0, _ = inputs.make_hidden(32768, dims.d_model, seed=0, device=DEV)
    Hg, idx, delta, K = _prefill(stack, h0, halt_layer=11, mode=mode, keep=0.5)
    assert K == 16384
    assert np.all(np.diff(idx) > 0)
    assert np.array_equal(idx, O.select_topk(delta.astype(np.float64), 0.5))
    out = Hg[:K] if mode == "prune" else Hg
    assert torch.isfinite(out.float()).all()
    del stack
    torch.cuda.empty_cache()


# ------------------------------------------------------- varlen batches
CU_TINY = [0, 200, 201, 512, 641]   # ragged lengths, one of a single token


def _prefill_varlen(stack, h0, cu, **kw):
    H = h0.to(DEV).clone()
    T = H.shape[0]
    idx = torch.full((T,), -1, dtype=torch.int32, device=DEV)
    delta = torch.empty(T, dtype=torch.float32, device=DEV)
    K, counts = dash.prefill_varlen(stack, H, cu, dash.make_config(**kw), idx_out=idx, delta_out=delta)
    assert dash.device_error() == 0
    return H.cpu(), idx[:K].cpu().numpy(), delta.cpu().numpy(), K, counts


@pytest.fixture(scope="module")
def tiny_varlen(tiny):
    dims, _, stack, L = tiny
    h0, _ = inputs.make_hidden(CU_TINY[-1], dims.d_model, seed=9)
    return dims, h0, stack, L


@pytest.mark.parametrize("mode", ["prune", "halt"])
@pytest.mark.parametrize("keep,nf,nl", [(0.5, 0, 0), (0.4, 16, 8)])
def test_prefill_varlen_tiny_matches_oracle(tiny_varlen, mode, keep, nf, nl):
    dims, h0, stack, L = tiny_varlen
    Hg, idx, delta, K, counts = _prefill_varlen(stack, h0, CU_TINY, halt_layer=1, mode=mode, keep=keep,
                                                keep_first=nf, keep_last=nl)
    free = O.dash_prefill_varlen(to_np(h0), CU_TINY, L, dims.as_dict(), 1, mode, keep=keep, keep_first=nf,
                                 keep_last=nl)
    assert counts == free["counts"] and K == sum(counts)
    assert _rel(delta, free["delta"]) < DELTA_TOL
    for s in range(len(CU_TINY) - 1):
        a, b = CU_TINY[s], CU_TINY[s + 1]
        mine = idx[(idx >= a) & (idx < b)]
        assert np.array_equal(mine - a, O.select_topk(delta[a:b].astype(np.float64), keep, nf, nl))
        ref = free["idx"][(free["idx"] >= a) & (free["idx"] < b)]
        _check_sets(mine, ref, free["delta"], _topk_cut(free["delta"][a:b], keep, nf, nl))
    assert np.array_equal(idx, free["idx"])
    got = to_np(Hg[:K]) if mode == "prune" else to_np(Hg)
    assert row_rel_err(got, free["hidden"]) < HIDDEN_TOL


def test_prefill_varlen_tiny_dense_and_threshold(tiny_varlen):
    dims, h0, stack, L = tiny_varlen
    Hd, _, _, K, counts = _prefill_varlen(stack, h0, CU_TINY, mode="dense")
    assert K == CU_TINY[-1] and counts == list(np.diff(CU_TINY))
    ref = O.dash_prefill_varlen(to_np(h0), CU_TINY, L, dims.as_dict(), 0, "halt", keep=1.0)
    dense = np.concatenate([O.dense_forward(to_np(h0)[a:b], L, dims.as_dict())
                            for a, b in zip(CU_TINY[:-1], CU_TINY[1:])])
    assert row_rel_err(to_np(Hd), dense) < HIDDEN_TOL
    thr = _clear_threshold(ref["delta"], 0.6)
    Hg, idx, delta, K, counts = _prefill_varlen(stack, h0, CU_TINY, halt_layer=0, mode="halt", select="threshold",
                                                threshold=thr)
    assert np.array_equal(idx, O.select_threshold(delta.astype(np.float64), np.float32(thr)))
    free = O.dash_prefill_varlen(to_np(h0), CU_TINY, L, dims.as_dict(), 0, "halt", select="threshold",
                                 threshold=thr)
    assert np.array_equal(idx, free["idx"])
    assert row_rel_err(to_np(Hg), free["hidden"]) < HIDDEN_TOL


def test_varlen_single_sequence_is_bitwise_plain_prefill(tiny):
    dims, h0, stack, L = tiny
    Ha, ia, da, Ka = _prefill(stack, h0, halt_layer=2, mode="prune", keep=0.5)
    Hb, ib, db, Kb, _ = _prefill_varlen(stack, h0, [0, 512], halt_layer=2, mode="prune", keep=0.5)
    assert Ka == Kb and np.array_equal(ia, ib) and np.array_equal(da, db) and torch.equal(Ha[:Ka], Hb[:Kb])


@pytest.mark.slow
def test_llama_varlen_two_layers_matches_oracle(gpu_lib):
    dims = inputs.LLAMA8B
    layers = inputs.make_layers(dims, seed=5, n_layers=2)
    stack = dash.Stack(dims, _dev_layers(layers))
    cu = [0, 256, 512, 640, 1024]
    h0, _ = inputs.make_varlen_hidden(n_seq=4, seq_len=256, text_len=64, d=dims.d_model, seed=5)
    Hg, idx, delta, K, counts = _prefill_varlen(stack, h0, cu, halt_layer=0, mode="prune", keep=0.4)
    L = layers_np(layers)
    free = O.dash_prefill_varlen(to_np(h0), cu, L, dims.as_dict(), 0, "prune", keep=0.4)
    assert counts == [math.floor(0.4 * n) for n in np.diff(cu)] == free["counts"]
    assert _rel(delta, free["delta"]) < DELTA_TOL
    assert np.array_equal(idx, free["idx"])
    assert row_rel_err(to_np(Hg[:K]), free["hidden"]) < HIDDEN_TOL


@pytest.mark.slow
def test_llama_varlen_4x16k_properties(gpu_lib):
    """The varlen workload: Llama-3.1-8B-shaped, 4 x 16384 tokens, halt at 13, keep 0.4, prune."""
    dims = inputs.LLAMA8B
    stack = dash.Stack(dims, inputs.make_layers(dims, seed=0, device=DEV))
    h0, cu = inputs.make_varlen_hidden(device=DEV)
    cu = cu.tolist()
    Hg, idx, delta, K, counts = _prefill_varlen(stack, h0, cu, halt_layer=13, mode="prune", keep=0.4)
    assert counts == [6553] * 4 and K == 4 * 6553
    for s in range(4):
        a, b = cu[s], cu[s + 1]
        mine = idx[(idx >= a) & (idx < b)]
        assert np.array_equal(mine - a, O.select_topk(delta[a:b].astype(np.float64), 0.4))
    assert torch.isfinite(Hg[:K].float()).all()
    del stack
    torch.cuda.empty_cache()


@pytest.mark.parametrize("mode,select,W", [("halt", "threshold", 2), ("prune", "topk", 3), ("prune", "threshold", 3)])
def test_prefill_monitor_window_matches_oracle(tiny, mode, select, W):
    dims, h0, stack, L = tiny
    base = O.dash_prefill(to_np(h0), L, dims.as_dict(), 2, mode, keep=1.0, monitor_layers=W)
    thr = _clear_threshold(base["delta"], 0.5)
    Hg, idx, delta, K = _prefill(stack, h0, halt_layer=2, mode=mode, select=select, keep=0.4, threshold=thr,
                                 monitor_layers=W)
    free = O.dash_prefill(to_np(h0), L, dims.as_dict(), 2, mode, select=select, keep=0.4, threshold=thr,
                          monitor_layers=W)
    assert _rel(delta, free["delta"]) < DELTA_TOL
    if select == "topk":
        assert np.array_equal(idx, O.select_topk(delta.astype(np.float64), 0.4))
        _check_sets(idx, free["idx"], free["delta"], _topk_cut(free["delta"], 0.4))
    else:
        assert np.array_equal(idx, O.select_threshold(delta.astype(np.float64), np.float32(thr)))
        _check_sets(idx, free["idx"], free["delta"], thr)
    assert np.array_equal(idx, free["idx"])
    got = to_np(Hg[:K]) if mode == "prune" else to_np(Hg)
    assert row_rel_err(got, free["hidden"]) < HIDDEN_TOL


@pytest.mark.parametrize("T", [1, 2, 127, 129, 300])
@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_prefill_ragged_lengths_match_oracle(tiny, T, mode):
    # degenerate and ragged prompts: a single token (K = 0), one tile +/- 1 row
    dims, h0, stack, L = tiny
    h = h0[:T]
    Hg, idx, delta, K = _prefill(stack, h, halt_layer=1, mode=mode, keep=0.5)
    free = O.dash_prefill(to_np(h), L, dims.as_dict(), 1, mode, keep=0.5)
    assert K == len(free["idx"]) == math.floor(0.5 * T)
    assert np.array_equal(idx, free["idx"])
    assert _rel(delta, free["delta"]) < DELTA_TOL
    got = to_np(Hg[:K]) if mode == "prune" else to_np(Hg)
    if len(got):
        assert row_rel_err(got, free["hidden"]) < HIDDEN_TOL


@pytest.mark.slow
def test_qwen_prefill_128k_threshold_halt_properties(gpu_lib):
    """The 128K workload's configuration (halt mode, relative Δ, threshold): the
    kept set is exactly {t : Δ_t >= thr} on the GPU's own Δ, halted rows equal
    the halting layer's output, and every output row is finite."""
    dims = inputs.QWEN7B
    T = 131072
    stack = dash.Stack(dims, inputs.make_layers(dims, seed=0, device=DEV, n_layers=3))
    h0, _ = inputs.make_hidden(T, dims.d_model, seed=0, device=DEV, span_rows=6528, span_len=128)
    Hg, idx, delta, K = _prefill(stack, h0, halt_layer=1, mode="halt", select="threshold", threshold=0.05,
                                 relative=True)
    assert np.array_equal(idx, O.select_threshold(delta.astype(np.float64), np.float32(0.05)))
    assert 0 < K < T
    first2 = dash.Stack(dims, inputs.make_layers(dims, seed=0, device=DEV, n_layers=2))
    Hs, _, _, _ = _prefill(first2, h0, mode="dense")
    halted = np.setdiff1d(np.arange(T), idx)
    assert torch.equal(Hg[halted], Hs[halted])
    assert torch.isfinite(Hg.float()).all()
    del stack, first2
    torch.cuda.empty_cache()
