"""GPU parity of the building-block kernels against the CPU oracle, through the C ABI."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as O
from long_context_prefill_tcgen05_b200 import dash, inputs
from conftest import to_np, row_rel_err, elem_rel_err, DELTA_TOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _no_device_error():
    assert dash.device_error() == 0


# ------------------------------------------------------------------ score
@pytest.mark.parametrize("relative", [False, True])
@pytest.mark.parametrize("T,d", [(1, 256), (777, 3584), (4096, 4096)])
def test_score_matches_oracle(gpu_lib, T, d, relative):
    U, H, _ = inputs.make_score_bench_inputs(T=T, d=d, seed=3)
    got = dash.score(U.to(DEV), H.to(DEV), relative=relative).cpu().numpy()
    ref = O.delta_scores(to_np(U), to_np(H), relative)
    assert np.max(np.abs(got - ref) / ref) < 1e-5  # fp32 sums of bf16 values
    assert np.max(np.abs(got - ref) / ref) < DELTA_TOL
    _no_device_error()


# ----------------------------------------------------------------- select
KINDS = ["random", "all_equal", "few_values", "signed_zero", "denormal", "negative", "spiky", "narrow"]


def _check_select(s, kind, keep=0.5, thr=0.0, nf=0, nl=0):
    sd = s.to(DEV)
    idx, halted, n = dash.select(sd, kind, keep, thr, nf, nl, want_halted=True)
    ref = (O.select_topk(s.double().numpy(), keep, nf, nl) if kind == "topk"
           else O.select_threshold(s.double().numpy(), float(np.float32(thr)), nf, nl))
    got = idx.cpu().numpy()
    assert n == len(ref)
    assert np.array_equal(got, ref)
    comp = np.setdiff1d(np.arange(len(s)), ref)
    assert np.array_equal(halted.cpu().numpy(), comp)


@pytest.mark.parametrize("pattern", KINDS)
@pytest.mark.parametrize("T", [1, 33, 1000, 1025, 4097, 32768, 100003, 131072])
def test_select_topk_bit_exact(gpu_lib, pattern, T):
    s = inputs.adversarial_scores(pattern, T, seed=T)
    for keep in (0.0, 1.0 / T, 0.5, 0.9, (T - 1) / T, 1.0):
        _check_select(s, "topk", keep)
    _check_select(s, "topk", 0.5, nf=64, nl=32)
    _check_select(s, "topk", 0.3, nf=T, nl=5)
    _no_device_error()


@pytest.mark.parametrize("pattern", KINDS)
@pytest.mark.parametrize("T", [1, 1000, 32768, 131072])
def test_select_threshold_bit_exact(gpu_lib, pattern, T):
    s = inputs.adversarial_scores(pattern, T, seed=T + 1)
    vals = s.numpy()
    for thr in (float(np.median(vals)), float(vals.max()), 0.0, float(vals[T // 2])):
        _check_select(s, "threshold", thr=thr)
    _check_select(s, "threshold", thr=float(np.median(vals)), nf=10, nl=10)
    _no_device_error()


def test_select_nonfinite_is_an_error(gpu_lib):
    for bad in (float("nan"), float("inf"), -float("inf")):
        s = torch.rand(5000)
        s[1234] = bad
        with pytest.raises(dash.DashError) as e:
            dash.select(s.to(DEV), "topk", 0.5)
        assert e.value.status == 3
        assert dash.device_error() == 3  # reported and cleared
    _no_device_error()


def test_select_empty(gpu_lib):
    idx, _, n = dash.select(torch.empty(0, device=DEV), "topk", 0.5)
    assert n == 0


# ------------------------------------------------------- compact / scatter
@pytest.mark.parametrize("T,d,K", [(1, 256, 1), (5000, 3584, 2500), (33000, 4096, 7)])
def test_compact_scatter_bit_exact(gpu_lib, T, d, K):
    g = torch.Generator().manual_seed(T)
    X = torch.randn(T, d, generator=g).to(torch.bfloat16)
    idx = torch.sort(torch.randperm(T, generator=g)[:K]).values.to(torch.int32)
    Y = dash.compact(X.to(DEV), idx.to(DEV))
    assert torch.equal(Y.cpu(), X[idx.long()])
    Z = X.clone().to(DEV)
    dash.scatter((Y * 2).contiguous(), idx.to(DEV), Z)
    ref = X.clone()
    ref[idx.long()] = X[idx.long()] * 2
    assert torch.equal(Z.cpu(), ref)
    _no_device_error()


def test_compact_bad_index_sets_device_error(gpu_lib):
    X = torch.randn(100, 256, device=DEV).to(torch.bfloat16)
    idx = torch.tensor([3, 100], dtype=torch.int32, device=DEV)   # 100 is out of range
    dash.compact(X, idx)
    assert dash.device_error() == 7
    _no_device_error()


# ----------------------------------------------------------------- RMSNorm
@pytest.mark.parametrize("M,d", [(1, 256), (1000, 3584), (300, 4096)])
def test_rmsnorm_matches_oracle(gpu_lib, M, d):
    g = torch.Generator().manual_seed(M)
    X = (torch.randn(M, d, generator=g) * 3).to(torch.bfloat16)
    w = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16)
    got = dash.rmsnorm(X.to(DEV), w.to(DEV), 1e-6).cpu()
    ref = O.rms_norm(to_np(X), to_np(w), 1e-6)
    assert row_rel_err(to_np(got), ref) < 8e-3   # bf16 output rounding
    _no_device_error()


# ----------------------------------------------------------- tcgen05 GEMM
@pytest.mark.parametrize("M,K,N", [(128, 64, 128), (1, 256, 512), (300, 3584, 4608), (1000, 704, 256),
                                   (129, 18944, 256), (2048, 3584, 3584)])
def test_linear_matches_fp64(gpu_lib, M, K, N):
    g = torch.Generator().manual_seed(M * 7 + N)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    got = dash.linear(A.to(DEV), W.to(DEV)).cpu()
    ref = to_np(A) @ to_np(W).T
    assert elem_rel_err(to_np(got), ref) < 1e-2
    assert row_rel_err(to_np(got), ref) < 5e-3
    _no_device_error()


@pytest.mark.parametrize("M,K,N", [(16384, 256, 3584), (32768, 128, 3584), (9700, 512, 4608)])
def test_linear_last_wave_rectangle_matches_single_sm_tiles(gpu_lib, M, K, N):
    """Shapes whose last wave of SM-pair tiles is mostly idle (896 = 12 x 74 + 8,
    1792 = 24 x 74 + 16 and 684 = 9 x 74 + 18 pair tiles, the last with a
    ragged 38th row tile): those tiles run as a rectangle of 128 x 128
    single-SM tiles after the others.  Every element is still one tile's sum
    over k in the same order, so it equals the all-single-SM result."""
    g = torch.Generator().manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    prev = dash.set_gemm_pairs(True)
    try:
        pair = dash.linear(A, W).cpu()
        dash.set_gemm_pairs(False)
        single = dash.linear(A, W).cpu()
    finally:
        dash.set_gemm_pairs(prev)
    _no_device_error()
    diff = (pair.float() - single.float()).abs().max().item()
    print(f"M={M} N={N} K={K}: max |pair - single| = {diff}")
    assert diff == 0.0
    rows = np.unique(np.r_[0, M - 1, np.arange(M - 300, M), np.random.default_rng(0).choice(M, 200, replace=False)])
    ref = to_np(A.cpu())[rows] @ to_np(W.cpu()).T
    assert row_rel_err(to_np(pair)[rows], ref) < 5e-3


@pytest.mark.parametrize("M,K,N", [(129, 64, 256), (300, 3584, 4608), (1000, 18944, 512), (4096, 3584, 4608),
                                   (8192, 3584, 3584)])
def test_linear_pair_tiles_match_fp64_and_single_sm_tiles(gpu_lib, M, K, N):
    """256x256 tiles on SM pairs (ragged last pair tile, a pair whose odd CTA
    has no live rows, more tiles than pairs, long K) against fp64 and against
    the single-SM kernel on the same inputs."""
    g = torch.Generator().manual_seed(M * 13 + N)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    prev = dash.set_gemm_pairs(True)
    try:
        pair = dash.linear(A, W).cpu()
        dash.set_gemm_pairs(False)
        single = dash.linear(A, W).cpu()
    finally:
        dash.set_gemm_pairs(prev)
    ref = to_np(A.cpu()) @ to_np(W.cpu()).T
    for got in (pair, single):
        assert elem_rel_err(to_np(got), ref) < 1e-2
        assert row_rel_err(to_np(got), ref) < 5e-3
    assert row_rel_err(to_np(pair), to_np(single).astype(np.float64)) < 1e-3
    _no_device_error()


# -------------------------------------------------------------- attention
def _attn_case(M, T_kv, hq, hkv, hd, qpos, seed):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(M, hq * hd, generator=g).to(torch.bfloat16)
    K = torch.randn(T_kv, hkv * hd, generator=g).to(torch.bfloat16)
    V = torch.randn(T_kv, hkv * hd, generator=g).to(torch.bfloat16)
    qp = None if qpos is None else torch.tensor(qpos, dtype=torch.int32)
    got = dash.attention(Q.to(DEV), K.to(DEV), V.to(DEV), hq, hkv, hd,
                         None if qp is None else qp.to(DEV)).cpu()
    q_pos = np.arange(M) if qpos is None else np.asarray(qpos)
    ref = O.causal_gqa_attention(to_np(Q).reshape(M, hq, hd), to_np(K).reshape(T_kv, hkv, hd),
                                 to_np(V).reshape(T_kv, hkv, hd), q_pos, np.arange(T_kv)).reshape(M, -1)
    return to_np(got), ref


@pytest.mark.parametrize("M,hq,hkv,hd", [(1, 4, 2, 64), (300, 4, 2, 64), (128, 7, 1, 128), (700, 28, 4, 128),
                                         (1030, 8, 2, 128)])
def test_attention_causal_matches_oracle(gpu_lib, M, hq, hkv, hd):
    got, ref = _attn_case(M, M, hq, hkv, hd, None, seed=M + hq)
    assert row_rel_err(got.reshape(M * hq, hd), ref.reshape(M * hq, hd)) < 2e-2
    assert elem_rel_err(got, ref) < 2e-2
    _no_device_error()


@pytest.mark.parametrize("M,T_kv,hq,hkv,hd", [(150, 500, 4, 2, 64), (260, 2000, 7, 1, 128), (1, 300, 4, 2, 64)])
def test_attention_indexed_queries_match_oracle(gpu_lib, M, T_kv, hq, hkv, hd):
    rng = np.random.default_rng(M)
    qpos = np.sort(rng.choice(T_kv, M, replace=False))
    got, ref = _attn_case(M, T_kv, hq, hkv, hd, qpos, seed=T_kv)
    assert row_rel_err(got.reshape(M * hq, hd), ref.reshape(M * hq, hd)) < 2e-2
    _no_device_error()


@pytest.mark.parametrize("M,hq,hkv,hd,growth", [(700, 8, 2, 128, 0.002), (1030, 4, 2, 64, 0.003),
                                                 (600, 4, 1, 128, 0.02)])
def test_attention_growing_scores_rescale_matches_oracle(gpu_lib, M, hq, hkv, hd, growth):
    """Scores that grow along the keys (k_j = noise + growth * j * u, q_i = noise + u for one fixed
    direction u of norm sqrt(hd)) make a row's maximum climb tile after tile, so the online softmax
    has to move its reference and rescale O and l, the path that random N(0,1) inputs never reach.
    The case checks that the climb really passes the kernel's lazy-rescale margin of 2^8."""
    g = torch.Generator().manual_seed(M + hd)
    u = torch.randn(hd, generator=g)
    u = u / u.norm() * hd ** 0.5
    pos = torch.arange(M, dtype=torch.float32)
    Q = (torch.randn(M, hq, hd, generator=g) + u).reshape(M, hq * hd).to(torch.bfloat16)
    K = (torch.randn(M, hkv, hd, generator=g) + growth * pos[:, None, None] * u).reshape(M, hkv * hd)
    K = K.to(torch.bfloat16)
    V = torch.randn(M, hkv * hd, generator=g).to(torch.bfloat16)
    q, k = to_np(Q).reshape(M, hq, hd), to_np(K).reshape(M, hkv, hd)
    # some row's causal maximum (log2 units) rises by more than 8 from one 128-key tile to a later one
    s = np.einsum("ihd,jhd->hij", q[:, ::hq // hkv], k) / np.sqrt(hd) * np.log2(np.e)  # head h*G <-> kv head h
    s = np.where(np.arange(M)[None, :, None] >= np.arange(M)[None, None, :], s, -np.inf)
    first = s[:, :, :128].max(-1)
    assert np.nanmax(s.max(-1) - first) > 8.0
    got = to_np(dash.attention(Q.to(DEV), K.to(DEV), V.to(DEV), hq, hkv, hd).cpu())
    ref = O.causal_gqa_attention(q, k, to_np(V).reshape(M, hkv, hd), np.arange(M), np.arange(M)).reshape(M, -1)
    assert row_rel_err(got.reshape(M * hq, hd), ref.reshape(M * hq, hd)) < 2e-2
    assert elem_rel_err(got, ref) < 2e-2
    _no_device_error()


def test_exp2_fma_within_its_error_bound(gpu_lib):
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 1.0, -1.0, 7.999])])
    y = dash.exp2_fma(x.to(DEV)).cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    assert np.max(np.abs(y - ref) / ref) < 1e-4          # fitted cubic: 7.5e-5
    low = dash.exp2_fma(torch.tensor([-125.5, -127.0, -200.0, -float("inf")], device=DEV)).cpu().numpy()
    assert np.all(np.isfinite(low) & (low > 0) & (low < 1e-37))  # clamped far below any bf16 weight
    _no_device_error()


@pytest.mark.parametrize("hd,hq,hkv,cu", [(64, 4, 2, [0, 300, 301, 700, 1030]), (128, 8, 2, [0, 256, 512, 900]),
                                          (128, 4, 1, [0, 1, 129, 130, 400])])
def test_attention_block_diagonal_matches_per_sequence_oracle(gpu_lib, hd, hq, hkv, cu):
    T = cu[-1]
    g = torch.Generator().manual_seed(T + hd)
    Q = torch.randn(T, hq * hd, generator=g).to(torch.bfloat16)
    K = torch.randn(T, hkv * hd, generator=g).to(torch.bfloat16)
    V = torch.randn(T, hkv * hd, generator=g).to(torch.bfloat16)
    kstart = torch.tensor(np.repeat(cu[:-1], np.diff(cu)), dtype=torch.int32)
    got = to_np(dash.attention(Q.to(DEV), K.to(DEV), V.to(DEV), hq, hkv, hd, kstart=kstart.to(DEV)).cpu())
    ref = np.concatenate([
        O.causal_gqa_attention(to_np(Q[a:b]).reshape(b - a, hq, hd), to_np(K[a:b]).reshape(b - a, hkv, hd),
                               to_np(V[a:b]).reshape(b - a, hkv, hd), np.arange(b - a), np.arange(b - a)
                               ).reshape(b - a, -1)
        for a, b in zip(cu[:-1], cu[1:])])
    assert row_rel_err(got.reshape(T * hq, hd), ref.reshape(T * hq, hd)) < 2e-2
    _no_device_error()


def test_bounded_wait_gives_up_with_timeout_status(gpu_lib):
    """A kernel waits on an mbarrier that nothing arrives on: the bounded wait
    gives up (about 2 s), the TIMEOUT status reaches the host, and the
    context stays usable."""
    done = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert dash.lib().dash_selftest_wait_timeout(ctypes.c_void_p(done.data_ptr())) == 6
    assert int(done.item()) == 2
    assert dash.device_error() == 0                      # read and cleared
    x = torch.randn(64, 256, device=DEV).to(torch.bfloat16)
    y = dash.rmsnorm(x, torch.ones(256, dtype=torch.bfloat16, device=DEV), 1e-6)  # still works
    assert torch.isfinite(y.float()).all()
