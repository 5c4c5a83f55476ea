"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: a library routine
(torch / transformers in fp64), a closed form, a brute-force enumeration, an
alternative formulation of the same definition, or values fixed by hand
from the pages (tests/golden).  A plausible slip in the oracle (dropped term,
wrong sign or index, transposed operand, wrong mask) fails at least one.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from long_context_prefill_tcgen05_b200 import inputs
from conftest import to_np, layers_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# --------------------------------------------------------------- block ops

def test_rms_norm_matches_torch():
    x = RNG.standard_normal((7, 96))
    g = RNG.standard_normal(96)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (96,), torch.tensor(g), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(x, g, 1e-6), ref, rtol=1e-13, atol=1e-13)


def test_rope_is_complex_rotation_of_each_pair():
    # pair (x_i, x_{i+hd/2}) as the complex number x_i + j x_{i+hd/2},
    # multiplied by exp(j * pos * theta^(-2i/hd)).
    n, nh, hd, theta = 5, 3, 16, 1e4
    x = RNG.standard_normal((n, nh, hd))
    pos = np.array([0, 1, 7, 1000, 131071])
    z = x[..., : hd // 2] + 1j * x[..., hd // 2:]
    i = np.arange(hd // 2)
    rot = np.exp(1j * pos[:, None, None] * theta ** (-2.0 * i / hd))
    zr = z * rot
    ref = np.concatenate([zr.real, zr.imag], axis=-1)
    np.testing.assert_allclose(O.apply_rope(x, pos, theta), ref, rtol=1e-10, atol=1e-10)


def test_rope_scores_depend_only_on_relative_position():
    hd, theta = 32, 1e6
    q = RNG.standard_normal((1, 1, hd))
    k = RNG.standard_normal((1, 1, hd))
    def dot(m, n):
        return float(np.sum(O.apply_rope(q, [m], theta) * O.apply_rope(k, [n], theta)))
    base = dot(40, 13)
    for s in (1, 77, 5000):
        assert math.isclose(dot(40 + s, 13 + s), base, rel_tol=1e-9, abs_tol=1e-9)
    # position 0 is the identity; rotation preserves norms
    np.testing.assert_allclose(O.apply_rope(q, [0], theta), q, rtol=0, atol=0)
    assert math.isclose(np.linalg.norm(O.apply_rope(q, [12345], theta)), np.linalg.norm(q), rel_tol=1e-12)


@pytest.mark.parametrize("hq,hkv", [(4, 2), (7, 1), (4, 4)])
def test_attention_matches_torch_sdpa(hq, hkv):
    n, hd = 37, 16
    q = RNG.standard_normal((n, hq, hd))
    k = RNG.standard_normal((n, hkv, hd))
    v = RNG.standard_normal((n, hkv, hd))
    pos = np.arange(n)
    got = O.causal_gqa_attention(q, k, v, pos, pos)
    tq, tk, tv = (torch.tensor(a).transpose(0, 1)[None] for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, enable_gqa=True)
    np.testing.assert_allclose(got, ref[0].transpose(0, 1).numpy(), rtol=1e-11, atol=1e-12)


def test_attention_position_mask_matches_sdpa_with_explicit_mask():
    # queries at sorted positions drawn from 0..m-1, keys at every position:
    # the halt-mode shape (compacted queries over all keys)
    m, hq, hkv, hd = 50, 4, 2, 8
    q_pos = np.sort(RNG.choice(m, 17, replace=False))
    q = RNG.standard_normal((17, hq, hd))
    k = RNG.standard_normal((m, hkv, hd))
    v = RNG.standard_normal((m, hkv, hd))
    got = O.causal_gqa_attention(q, k, v, q_pos, np.arange(m))
    mask = torch.tensor(np.arange(m)[None, :] <= q_pos[:, None])
    tq, tk, tv = (torch.tensor(a).transpose(0, 1)[None] for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, enable_gqa=True)
    np.testing.assert_allclose(got, ref[0].transpose(0, 1).numpy(), rtol=1e-11, atol=1e-12)


def test_attention_closed_forms():
    n, hd = 9, 4
    k = np.ones((n, 1, hd))                 # equal scores -> causal running mean of V
    v = RNG.standard_normal((n, 1, hd))
    q = RNG.standard_normal((n, 2, hd))
    got = O.causal_gqa_attention(q, k, v, np.arange(n), np.arange(n))
    cum = np.cumsum(v[:, 0, :], axis=0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(got[:, 0, :], cum, rtol=1e-12)
    np.testing.assert_allclose(got[:, 1, :], cum, rtol=1e-12)
    # one dominant key: a huge logit selects that key's value exactly
    k2 = np.zeros((n, 1, hd)); k2[3, 0, 0] = 1e4
    q2 = np.zeros((n, 1, hd)); q2[:, 0, 0] = 1.0
    got2 = O.causal_gqa_attention(q2, k2, v, np.arange(n), np.arange(n))
    np.testing.assert_allclose(got2[3:, 0, :], np.repeat(v[3:4, 0, :], n - 3, 0), atol=1e-12)


def test_silu_matches_torch():
    x = RNG.standard_normal(100) * 5
    np.testing.assert_allclose(O.silu(x), torch.nn.functional.silu(torch.tensor(x)).numpy(), rtol=1e-13)


def _hf_llama(dims, layers_t, n_layers):
    """transformers' Llama decoder (fp64, eager attention, no final norm) loaded with our weights."""
    from transformers import LlamaConfig, LlamaModel
    cfg = LlamaConfig(hidden_size=dims.d_model, num_attention_heads=dims.n_heads,
                      num_key_value_heads=dims.n_kv_heads, head_dim=dims.head_dim,
                      intermediate_size=dims.ffn_dim, num_hidden_layers=n_layers,
                      rms_norm_eps=dims.rms_eps, vocab_size=8,
                      rope_parameters={"rope_type": "default", "rope_theta": dims.rope_theta},
                      max_position_embeddings=1 << 18, attn_implementation="eager")
    model = LlamaModel(cfg).double().eval()
    model.norm = torch.nn.Identity()
    with torch.no_grad():
        for lay, w in zip(model.layers, layers_t):
            lay.self_attn.q_proj.weight.copy_(w["wq"].double())
            lay.self_attn.k_proj.weight.copy_(w["wk"].double())
            lay.self_attn.v_proj.weight.copy_(w["wv"].double())
            lay.self_attn.o_proj.weight.copy_(w["wo"].double())
            lay.mlp.gate_proj.weight.copy_(w["wg"].double())
            lay.mlp.up_proj.weight.copy_(w["wu"].double())
            lay.mlp.down_proj.weight.copy_(w["wd"].double())
            lay.input_layernorm.weight.copy_(w["attn_norm"].double())
            lay.post_attention_layernorm.weight.copy_(w["ffn_norm"].double())
    return model


# transformers evaluates the rotary angles in fp32 (about 1e-7 relative), so
# these comparisons allow 1e-6; a structural slip shows up at 1e-2 or more.
HF_TOL = dict(rtol=1e-6, atol=1e-6)


def _hf_run(model, h, pos):
    with torch.no_grad():
        out = model(inputs_embeds=torch.tensor(h)[None], position_ids=torch.tensor(pos)[None])
    return out.last_hidden_state[0].numpy()


def test_decoder_stack_matches_transformers_llama():
    dims = inputs.TINY
    layers_t = inputs.make_layers(dims, seed=3, n_layers=2)
    # non-trivial norm gains so a dropped gain is caught
    gen = torch.Generator().manual_seed(7)
    for w in layers_t:
        w["attn_norm"] = (1 + 0.1 * torch.randn(dims.d_model, generator=gen)).to(torch.bfloat16)
        w["ffn_norm"] = (1 + 0.1 * torch.randn(dims.d_model, generator=gen)).to(torch.bfloat16)
    h0 = to_np(inputs.make_hidden(96, dims.d_model, seed=5)[0])
    got = O.dense_forward(h0, layers_np(layers_t), dims.as_dict())
    ref = _hf_run(_hf_llama(dims, layers_t, 2), h0, np.arange(96))
    np.testing.assert_allclose(got, ref, **HF_TOL)


# ------------------------------------------------------------ prefill pins

@pytest.fixture(scope="module")
def tiny_np(tiny_stack):
    dims, layers, h0 = tiny_stack
    return dims.as_dict(), layers_np(layers), to_np(h0), layers


def test_prune_equals_transformers_on_kept_subsequence(tiny_np, tiny_stack):
    dims_d, L, h0, layers_t = tiny_np
    dims = tiny_stack[0]
    r = O.dash_prefill(h0, L, dims_d, halt_layer=1, mode="prune", keep=0.5)
    idx = r["idx"]
    assert len(idx) == 256
    ref = _hf_run(_hf_llama(dims, layers_t[2:], 2), r["halt_out"][idx], idx)
    np.testing.assert_allclose(r["hidden"], ref, **HF_TOL)


@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_keep_one_equals_dense(tiny_np, mode):
    dims_d, L, h0, _ = tiny_np
    h = h0[:128]
    r = O.dash_prefill(h, L, dims_d, halt_layer=2, mode=mode, keep=1.0)
    assert np.array_equal(r["idx"], np.arange(128))
    np.testing.assert_allclose(r["hidden"], O.dense_forward(h, L, dims_d), rtol=1e-12, atol=1e-12)


def test_halting_layer_output_independent_of_keep(tiny_np):
    dims_d, L, h0, _ = tiny_np
    h = h0[:160]
    a = O.dash_prefill(h, L, dims_d, halt_layer=2, mode="prune", keep=0.25)
    b = O.dash_prefill(h, L, dims_d, halt_layer=2, mode="halt", keep=0.75)
    assert np.array_equal(a["halt_out"], b["halt_out"])
    assert np.array_equal(a["delta"], b["delta"])


def test_delta_is_norm_of_attention_update(tiny_np):
    # With the FFN's down projection zeroed the block returns H' = H + U, so
    # ||block(H) - H|| must equal the oracle's Δ from U.
    dims_d, L, h0, _ = tiny_np
    h = h0[:96]
    pos = np.arange(96)
    w = dict(L[0]); w["wd"] = np.zeros_like(w["wd"])
    out, u = O.decoder_block(h, pos, h, pos, w, dims_d)
    direct = np.linalg.norm(out - h, axis=1)
    np.testing.assert_allclose(O.delta_scores(u), direct, rtol=1e-12)
    rel = O.delta_scores(u, h, relative=True)
    np.testing.assert_allclose(rel, direct / np.linalg.norm(h, axis=1), rtol=1e-12)


def test_halt_mode_equals_dense_with_restore(tiny_np):
    # Alternative formulation of halt mode: run each later layer densely on
    # all rows, then put the halted rows back to their frozen state.
    dims_d, L, h0, _ = tiny_np
    h = h0[:200]
    r = O.dash_prefill(h, L, dims_d, halt_layer=1, mode="halt", keep=0.4)
    idx = r["idx"]
    halted = np.setdiff1d(np.arange(200), idx)
    state = r["halt_out"].copy()
    for l in range(2, len(L)):
        state = O.dense_forward(state, [L[l]], dims_d)
        state[halted] = r["halt_out"][halted]
    np.testing.assert_allclose(r["hidden"], state, rtol=1e-11, atol=1e-11)
    # halted rows are bit-identical to the halting layer's output
    assert np.array_equal(r["hidden"][halted], r["halt_out"][halted])


def test_prefill_topk_count_and_order(tiny_np):
    dims_d, L, h0, _ = tiny_np
    r = O.dash_prefill(h0[:100], L, dims_d, halt_layer=0, mode="prune", keep=0.37)
    assert len(r["idx"]) == math.floor(0.37 * 100)
    assert np.all(np.diff(r["idx"]) > 0)


# ---------------------------------------------------------------- selection

def _brute_topk(scores, k):
    """Token t is chosen iff fewer than k tokens beat it, where s beats t when
    score_s > score_t, or score_s == score_t and s < t."""
    T = len(scores)
    out = []
    for t in range(T):
        beaten_by = sum(1 for s in range(T)
                        if scores[s] > scores[t] or (scores[s] == scores[t] and s < t))
        if beaten_by < k:
            out.append(t)
    return np.array(out, dtype=np.int64)


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_select_topk_all_tie_patterns_brute_force(T):
    # every score vector over a 3-value alphabet (ties everywhere) and every keep
    for vals in itertools.product([0.0, 0.5, 1.0], repeat=T):
        s = np.array(vals)
        for k in range(T + 1):
            keep = k / T
            assert O.topk_count(T, keep) == k
            got = O.select_topk(s, keep)
            assert np.array_equal(got, _brute_topk(s, k)), (vals, k)


def test_select_topk_is_a_top_set_of_every_subset():
    # the chosen set is the unique size-k set in which every member beats
    # every non-member under (score desc, index asc)
    s = np.array([0.3, 0.9, 0.3, 0.1, 0.9, 0.5, 0.3])
    T, k = len(s), 4
    key = lambda t: (-s[t], t)
    winners = [set(c) for c in itertools.combinations(range(T), k)
               if all(key(a) < key(b) for a in c for b in set(range(T)) - set(c))]
    assert len(winners) == 1
    assert set(O.select_topk(s, k / T).tolist()) == winners[0]


def test_select_topk_random_large_matches_brute_force():
    s = np.round(RNG.random(300), 2)       # many ties
    for keep in (0.0, 0.1, 0.5, 0.99, 1.0):
        k = math.floor(keep * 300)
        assert np.array_equal(O.select_topk(s, keep), _brute_topk(s, k))


def test_select_signed_zero_is_a_tie():
    s = np.array([0.0, -0.0, 0.0, -0.0, 1.0])
    assert np.array_equal(O.select_topk(s, 0.6), [0, 1, 4])


@pytest.mark.parametrize("T,nf,nl,keep", [(40, 4, 3, 0.5), (10, 6, 6, 0.5), (30, 0, 5, 0.2),
                                          (30, 5, 0, 0.9), (7, 0, 0, 1.0)])
def test_forced_first_last(T, nf, nl, keep):
    s = RNG.random(T)
    got = O.select_topk(s, keep, nf, nl)
    forced = [t for t in range(T) if t < nf or (nl > 0 and t >= T - nl)]
    mid = [t for t in range(T) if t not in forced]
    k_dyn = math.floor(keep * len(mid))
    best_mid = sorted(mid, key=lambda t: (-s[t], t))[:k_dyn]
    assert got.tolist() == sorted(forced + best_mid)
    assert O.topk_count(T, keep, nf, nl) == len(got)


def test_select_threshold_brute_force():
    s = np.round(RNG.random(64), 1)
    for thr in (0.0, 0.3, 0.5, 1.0, 2.0):
        got = O.select_threshold(s, thr, 2, 1)
        ref = [t for t in range(64) if s[t] >= thr or t < 2 or t == 63]
        assert got.tolist() == ref


def test_nonfinite_scores_raise():
    for bad in (np.nan, np.inf, -np.inf):
        s = np.ones(8); s[3] = bad
        with pytest.raises(O.OracleError):
            O.select_topk(s, 0.5)
        with pytest.raises(O.OracleError):
            O.select_threshold(s, 0.5)
    with pytest.raises(O.OracleError):
        O.delta_scores(np.ones((2, 3)), np.zeros((2, 3)), relative=True)


def test_gather_scatter_roundtrip():
    x = RNG.standard_normal((20, 3))
    idx = np.array([1, 4, 5, 19])
    y = O.gather_rows(x, idx) * 2
    z = O.scatter_rows(x, y, idx)
    assert np.array_equal(z[idx], 2 * x[idx])
    rest = np.setdiff1d(np.arange(20), idx)
    assert np.array_equal(z[rest], x[rest])


# ------------------------------------------------------------------ golden

def _read_golden(name):
    cases = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                cases.append([field.strip() for field in line.split("|")])
    return cases


def test_golden_selection_worked_examples():
    for scores, keep, nf, nl, expect in _read_golden("select_worked.txt"):
        s = np.array([float(v) for v in scores.split()])
        got = O.select_topk(s, float(keep), int(nf), int(nl))
        assert got.tolist() == [int(v) for v in expect.split()], (scores, keep)


def test_golden_counts_from_the_pages():
    for kind, args, expect in _read_golden("counts.txt"):
        a = [float(v) for v in args.split()]
        if kind == "halt_layer":        # L_s = floor(0.4 * total layers)
            got = math.floor(a[0] * a[1])
        else:                           # K_effective
            T, keep, nf, nl = int(a[0]), a[1], int(a[2]), int(a[3])
            got = O.topk_count(T, keep, nf, nl)
        assert got == int(expect), (kind, args)


def test_varlen_oracle_is_per_sequence_and_order_independent(tiny_np):
    dims_d, L, h0, _ = tiny_np
    cu = [0, 70, 71, 200]
    r = O.dash_prefill_varlen(h0[:200], cu, L, dims_d, 1, "prune", keep=0.5)
    assert r["counts"] == [35, 0, 64]            # floor(0.5 * len) per sequence
    # each sequence is the single-sequence prefill of its own rows
    one = O.dash_prefill(h0[71:200], L, dims_d, 1, "prune", keep=0.5)
    np.testing.assert_array_equal(r["idx"][35:], one["idx"] + 71)
    np.testing.assert_allclose(r["hidden"][35:], one["hidden"], rtol=0, atol=0)
    # swapping the sequences swaps the results: nothing crosses a boundary
    sw = np.concatenate([h0[71:200], h0[0:71]])
    r2 = O.dash_prefill_varlen(sw, [0, 129, 199, 200], L, dims_d, 1, "prune", keep=0.5)
    np.testing.assert_allclose(r2["hidden"][:64], r["hidden"][35:], rtol=0, atol=0)
    np.testing.assert_allclose(r2["hidden"][64:], r["hidden"][:35], rtol=0, atol=0)


def test_consecutive_layer_monitoring_brute_force(tiny_np):
    # halted = tokens whose update is below the threshold in EVERY monitored
    # layer, computed from per-layer deltas of directly run blocks
    dims_d, L, h0, _ = tiny_np
    h = h0[:150]
    pos = np.arange(150)
    per_layer, x = [], h
    for l in range(3):
        out, u = O.decoder_block(x, pos, x, pos, L[l], dims_d)
        per_layer.append(np.linalg.norm(u, axis=1))
        x = out
    thr = float(np.median(per_layer[2]))
    for W in (1, 2, 3):
        r = O.dash_prefill(h, L, dims_d, 2, "halt", select="threshold", threshold=thr, monitor_layers=W)
        stays = [t for t in range(150) if any(per_layer[l][t] >= thr for l in range(3 - W, 3))]
        assert r["idx"].tolist() == stays
    # top-k ranks by the window maximum
    r = O.dash_prefill(h, L, dims_d, 2, "prune", keep=0.3, monitor_layers=2)
    np.testing.assert_allclose(r["delta"], np.maximum(per_layer[1], per_layer[2]), rtol=1e-12)
    with pytest.raises(O.OracleError):
        O.dash_prefill(h, L, dims_d, 1, "prune", monitor_layers=3)


# ---------------------------------------------------------------- decode pins

def test_prefill_cache_and_decode_match_transformers_kv_cache():
    # transformers' own incremental decoding: its cache after the prompt and
    # the hidden state of one generated token, against the oracle's dense
    # prefill cache and dash_decode.
    dims = inputs.TINY
    layers_t = inputs.make_layers(dims, seed=3, n_layers=2)
    gen = torch.Generator().manual_seed(8)
    for w in layers_t:
        w["attn_norm"] = (1 + 0.1 * torch.randn(dims.d_model, generator=gen)).to(torch.bfloat16)
    L = layers_np(layers_t)
    h = to_np(inputs.make_hidden(49, dims.d_model, seed=6)[0])
    prompt, new = h[:48], h[48:]
    r = O.dash_prefill(prompt, L, dims.as_dict(), halt_layer=1, mode="prune", keep=1.0, return_kv=True)
    model = _hf_llama(dims, layers_t, 2)
    with torch.no_grad():
        out = model(inputs_embeds=torch.tensor(prompt)[None], position_ids=torch.arange(48)[None], use_cache=True)
        cache = out.past_key_values
        for l in range(2):
            k, v, p = r["kv"][l]
            assert np.array_equal(p, np.arange(48))
            # rotated keys carry the fp32 angle error (about 6e-8 x angle, angles
            # up to 47 rad here) times |k|: 1e-5 of max|k| bounds it; a wrong
            # pairing, sign or position is off by order |k|.
            ref_k = cache.layers[l].keys[0].numpy().transpose(1, 0, 2)
            np.testing.assert_allclose(k, ref_k, rtol=0, atol=1e-5 * np.abs(ref_k).max())
            np.testing.assert_allclose(v, cache.layers[l].values[0].numpy().transpose(1, 0, 2), **HF_TOL)
        step = model(inputs_embeds=torch.tensor(new)[None], position_ids=torch.tensor([[48]]),
                     past_key_values=cache, use_cache=True)
    got, _ = O.dash_decode(new, [48], r["kv"], L, dims.as_dict())
    np.testing.assert_allclose(got, step.last_hidden_state[0].numpy(), **HF_TOL)


def test_decode_equals_dense_forward_of_the_longer_sequence(tiny_np):
    # Two generated tokens on a dense cache, one at a time, are the last two
    # rows of a dense forward over prompt + both tokens.
    dims_d, L, h0, _ = tiny_np
    h = h0[:66]
    r = O.dash_prefill(h[:64], L, dims_d, halt_layer=len(L) - 1, mode="prune", keep=1.0, return_kv=True)
    y1, kv = O.dash_decode(h[64:65], [64], r["kv"], L, dims_d)
    y2, kv = O.dash_decode(h[65:66], [65], kv, L, dims_d)
    ref = O.dense_forward(h, L, dims_d)
    np.testing.assert_allclose(np.concatenate([y1, y2]), ref[64:], rtol=1e-11, atol=1e-11)
    # several new tokens in one call attend causally among themselves
    y12, _ = O.dash_decode(h[64:66], [64, 65], r["kv"], L, dims_d)
    np.testing.assert_allclose(y12, ref[64:], rtol=1e-11, atol=1e-11)
    assert all(len(k) == 66 for k, _, _ in kv)


@pytest.mark.parametrize("mode", ["prune", "halt"])
def test_decode_on_pruned_cache_equals_prefill_with_the_new_token_active(tiny_np, mode):
    # The generated token sees exactly what it would see as an extra active
    # token of a prefill over prompt + token: the same rows in layers
    # 0..L_s, and in later layers the active set (prune) or every row with
    # the halted ones frozen (halt).
    dims_d, L, h0, _ = tiny_np
    T = 120
    r = O.dash_prefill(h0[:T], L, dims_d, halt_layer=1, mode=mode, keep=0.4, return_kv=True)
    idx = r["idx"]
    K = len(idx)
    rows = [len(k) for k, _, _ in r["kv"]]
    late = K if mode == "prune" else T
    assert rows == [T, T, late, late]
    assert np.array_equal(r["kv"][2][2], idx if mode == "prune" else np.arange(T))
    got, kv = O.dash_decode(h0[T:T + 1], [T], r["kv"], L, dims_d)
    ext = O.dash_prefill(h0[:T + 1], L, dims_d, halt_layer=1, mode=mode,
                         forced_idx=np.concatenate([idx, [T]]))
    np.testing.assert_allclose(got, ext["hidden"][-1:], rtol=1e-11, atol=1e-11)
    assert [len(k) for k, _, _ in kv] == [T + 1, T + 1, late + 1, late + 1]


def test_varlen_prefill_returns_one_cache_per_sequence(tiny_np):
    dims_d, L, h0, _ = tiny_np
    cu = [0, 70, 70, 150]
    r = O.dash_prefill_varlen(h0[:150], cu, L, dims_d, halt_layer=2, keep=0.5, return_kv=True)
    assert r["kv"][1] is None
    for s, (a, b) in enumerate([(0, 70), (70, 150)]):
        kv = r["kv"][0 if s == 0 else 2]
        one = O.dash_prefill(h0[a:b], L, dims_d, halt_layer=2, keep=0.5, return_kv=True)
        for (k1, v1, p1), (k2, v2, p2) in zip(kv, one["kv"]):
            assert np.array_equal(k1, k2) and np.array_equal(v1, v2) and np.array_equal(p1, p2)
