"""Plain fp64 CPU oracle for Delta-Attention Selective Halting (DASH) prefill.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct
definition that the CUDA library is checked against.  Only the test suite,
the smoke check and the CPU-baseline legs of the benchmark may use it; the
product path never imports it.  It shares no code, tables or constants with
the CUDA library; both sides only consume the same seeded inputs.

Every array is float64; bf16 inputs are widened exactly before they reach
this module.  No blocking, fusion or reordering beyond the plain definitions:
numpy's matmul, sort and elementary functions are the only library steps.

Pages cited below (short name -> page title):
  [DASH blog]  "DASH：基于注意力增量的Transformer令牌压缩，实现长序列推理高效加速"
               (bbs.csdn.net).  §2.1 defines the attention update U and
               Δattn_t = ||U_t||_2; §2.3 single-shot halting at layer L_s;
               §3.1 the algorithm steps (top-K with K = floor((1-ρ)·T),
               forced first/last tokens, K_effective, gather of S*);
               §3.2 parameter table; §3.3 the prefill pseudocode;
               §5.1 per-sample decisions in a batch.
  [DASH news]  "DASH：通过注意力动态监测实现长上下文高效预填充" (zingnex.cn).
               Section "层间更新动态监测": tokens whose update falls below a
               preset threshold are judged stable; section "选择性停止机制":
               halted tokens keep their KV-cache state but take no further
               self-attention compute.
  [DASH abs]   "Stability Implies Redundancy: Delta Attention Selective
               Halting for Efficient Long-Context Prefilling" (abstract).
  [DoSA]       "DoSA: Dots Sparse Attention: 中文精读笔记", §2.6 Theorem 1:
               an exact top-K id set needs one agreed tie order.

Readings taken where the pages are silent or garbled:
  R1 pre-norm block (norm -> attention -> U, H' = H + U, [DASH blog] §2.1);
     the pseudocode's norm-after-add in §3.3 is read as a simplification.
  R2 RMSNorm with eps given by the model dims (1e-6 for every workload here).
  R3 RoPE in rotate-half form: pairs (i, i + hd/2), angle pos·θ^(-2i/hd).
  R4 no biases in any projection.
  R5 U is the attention module output after o_proj, before the residual add.
  R6 the halting layer itself runs on all T tokens; selection follows it.
  R7 layers are numbered from 0; "halt at layer L_s" means layers 0..L_s run
     in full.
  R8 K = floor(keep·n) (floor of the product in double precision); K = 0 is
     allowed and yields an empty set.
  R9 ties are broken by the lower token index (the pages leave the order
     open; [DoSA] §2.6 explains why one fixed order is needed).
  R10 threshold selection keeps t iff Δ_t >= threshold.
  R11 keep_last = 0 protects no token (the pseudocode's [-0:] slice would
      mark the whole sequence, a garbled edge).
  R12 halt mode recomputes the K/V of halted rows in every later layer from
      their frozen hidden state with that layer's weights.
  R13 prune mode keeps each token's original position for RoPE; the causal
      order of the kept tokens is their original order.
  R14 a non-finite score (or ||H_t|| = 0 in relative mode) is an error, and
      no selection is made.
  R15 the relative score divides by the norm of the halting layer's input
      residual stream H.
  R17 generation after the prefill: the KV cache of a layer holds the keys
      and values that layer's attention read during the prefill; a generated
      token runs every layer and attends to that cache plus itself.
  R18 a generated token's RoPE position continues the original numbering
      (T for the first one after a T-token prompt), in prune mode too (R13).
  (R16 is a reading of the pages that concerns no oracle function.)
"""
import math

import numpy as np

__all__ = [
    "rms_norm", "rope_inv_freq", "apply_rope", "causal_gqa_attention", "silu",
    "swiglu", "decoder_block", "dense_forward", "delta_scores", "forced_mask",
    "topk_count", "select_topk", "select_threshold", "gather_rows",
    "scatter_rows", "dash_prefill", "dash_prefill_varlen", "layer_kv",
    "block_with_kv", "dash_decode", "OracleError",
]


class OracleError(ValueError):
    """Raised where the CUDA library returns an error status (R14)."""


# ---------------------------------------------------------------- block ops

def rms_norm(x, g, eps):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g (R1, R2)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def rope_inv_freq(head_dim, theta):
    """Rotary frequencies theta^(-2i/hd) for i in [0, hd/2) (R3)."""
    half = head_dim // 2
    return float(theta) ** (-(2.0 * np.arange(half, dtype=np.float64)) / head_dim)


def apply_rope(x, pos, theta):
    """Rotate-half RoPE (R3).

    x: [n, heads, hd]; pos: [n] integer positions.  Element i and element
    i + hd/2 of every head form a pair rotated by angle pos * inv_freq[i].
    """
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(hd, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def causal_gqa_attention(q, k, v, q_pos, k_pos):
    """Softmax attention with a position-causal mask and grouped KV heads.

    q: [n, hq, hd]; k, v: [m, hkv, hd].  Query i sees key j iff
    k_pos[j] <= q_pos[i].  Query head h reads KV head h // (hq / hkv).
    Scores are scaled by 1/sqrt(hd); the softmax subtracts the row maximum.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, hq, hd = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    visible = np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None]
    if not visible.any(axis=1).all():
        raise OracleError("a query row sees no key")
    out = np.empty((n, hq, hd), dtype=np.float64)
    scale = 1.0 / math.sqrt(hd)
    for h in range(hq):
        kv = h // group
        s = (q[:, h, :] @ k[:, kv, :].T) * scale
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, kv, :]
    return out


def silu(x):
    """x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def swiglu(gate, up):
    """SwiGLU activation silu(gate) * up."""
    return silu(gate) * up


def layer_kv(h_kv, kv_pos, w, dims):
    """Keys (RoPE applied at kv_pos) and values of the rows h_kv [m, d] for one
    layer: the entries a KV cache holds for them ([DASH blog] §2.1 block, R1-R4).
    Returns k, v of shape [m, hkv, hd]."""
    eps, theta = dims["rms_eps"], dims["rope_theta"]
    hkv, hd = dims["n_kv_heads"], dims["head_dim"]
    h_kv = np.asarray(h_kv, dtype=np.float64)
    a_kv = rms_norm(h_kv, w["attn_norm"], eps)
    k = apply_rope((a_kv @ w["wk"].T).reshape(len(h_kv), hkv, hd), kv_pos, theta)
    v = (a_kv @ w["wv"].T).reshape(len(h_kv), hkv, hd)
    return k, v


def block_with_kv(h_q, q_pos, k, v, kv_pos, w, dims):
    """The decoder block of the rows h_q (positions q_pos) attending to given
    keys/values k, v [m, hkv, hd] at positions kv_pos.  Returns (out, U) as
    decoder_block does."""
    eps, theta = dims["rms_eps"], dims["rope_theta"]
    hq, hd = dims["n_heads"], dims["head_dim"]
    h_q = np.asarray(h_q, dtype=np.float64)
    if len(h_q) == 0:  # no active rows: nothing to update
        return h_q.copy(), np.zeros_like(h_q)
    a_q = rms_norm(h_q, w["attn_norm"], eps)
    q = apply_rope((a_q @ w["wq"].T).reshape(len(h_q), hq, hd), q_pos, theta)
    o = causal_gqa_attention(q, k, v, q_pos, kv_pos).reshape(len(h_q), hq * hd)
    u = o @ w["wo"].T
    h1 = h_q + u
    b = rms_norm(h1, w["ffn_norm"], eps)
    f = swiglu(b @ w["wg"].T, b @ w["wu"].T) @ w["wd"].T
    return h1 + f, u


def decoder_block(h_q, q_pos, h_kv, kv_pos, w, dims):
    """One pre-norm decoder block ([DASH blog] §2.1; R1-R5).

    h_q: [n, d] rows that issue queries and are updated (positions q_pos).
    h_kv: [m, d] rows whose keys/values the queries attend to (positions
    kv_pos).  In a dense layer both are the same rows.

    Returns (out, U): out = H' + FFN(H'), H' = h_q + U, U = attention output
    after o_proj and before the residual add.
    """
    if len(h_q) == 0:
        h_q = np.asarray(h_q, dtype=np.float64)
        return h_q.copy(), np.zeros_like(h_q)
    k, v = layer_kv(h_kv, kv_pos, w, dims)
    return block_with_kv(h_q, q_pos, k, v, kv_pos, w, dims)


def dense_forward(h0, layers, dims, pos=None):
    """Run every layer on every row (no halting)."""
    h = np.asarray(h0, dtype=np.float64)
    pos = np.arange(len(h)) if pos is None else np.asarray(pos)
    for w in layers:
        h, _ = decoder_block(h, pos, h, pos, w, dims)
    return h


# ------------------------------------------------------------- score/select

def delta_scores(u, h_in=None, relative=False):
    """Δattn_t = ||U_t||_2 ([DASH blog] §2.1); relative form ||U_t||/||H_t|| (R15)."""
    u = np.asarray(u, dtype=np.float64)
    d = np.sqrt(np.sum(u * u, axis=1))
    if relative:
        hn = np.sqrt(np.sum(np.asarray(h_in, dtype=np.float64) ** 2, axis=1))
        if np.any(hn == 0.0):
            raise OracleError("||H_t|| = 0 in relative mode")
        d = d / hn
    return d


def forced_mask(T, keep_first=0, keep_last=0):
    """Tokens always kept: the first keep_first and the last keep_last
    ([DASH blog] §3.1 "重要细节"; R11 for keep_last = 0)."""
    t = np.arange(T)
    return (t < keep_first) | (t >= T - keep_last if keep_last > 0 else np.zeros(T, bool))


def topk_count(T, keep, keep_first=0, keep_last=0):
    """K_effective = |forced| + floor(keep · (tokens not forced)) ([DASH blog] §3.1, R8).

    With no forced tokens this is K = floor((1-ρ)·T), keep = 1-ρ.
    """
    nforced = int(forced_mask(T, keep_first, keep_last).sum())
    return nforced + math.floor(keep * (T - nforced))


def _check_finite(scores):
    if not np.all(np.isfinite(scores)):
        raise OracleError("non-finite score")


def select_topk(scores, keep, keep_first=0, keep_last=0):
    """Active set S*: forced tokens plus the floor(keep·n) highest-scoring
    other tokens, returned as ascending indices ([DASH blog] §3.1 and the
    final torch.sort of §3.3).  Order: score descending, then lower index
    first (R9)."""
    scores = np.asarray(scores, dtype=np.float64)
    _check_finite(scores)
    T = len(scores)
    forced = forced_mask(T, keep_first, keep_last)
    mid = np.flatnonzero(~forced)
    k_dyn = math.floor(keep * len(mid))
    # lexsort: last key is primary -> (-score ascending, index ascending).
    order = mid[np.lexsort((mid, -scores[mid]))]
    chosen = order[:k_dyn]
    return np.sort(np.concatenate([np.flatnonzero(forced), chosen])).astype(np.int64)


def select_threshold(scores, threshold, keep_first=0, keep_last=0):
    """Tokens with Δ_t >= threshold stay active ([DASH news] "层间更新动态监测";
    R10), plus forced tokens; ascending indices."""
    scores = np.asarray(scores, dtype=np.float64)
    _check_finite(scores)
    keep = forced_mask(len(scores), keep_first, keep_last) | (scores >= threshold)
    return np.flatnonzero(keep).astype(np.int64)


def gather_rows(x, idx):
    """Compaction: row i of the output is row idx[i] of x ([DASH blog] §3.1 "复用活跃集合")."""
    return np.asarray(x)[np.asarray(idx)]


def scatter_rows(x_full, y, idx):
    """Inverse of gather: x_full[idx[i]] = y[i]; other rows unchanged."""
    out = np.array(x_full, copy=True)
    out[np.asarray(idx)] = y
    return out


# ------------------------------------------------------------------ prefill

def dash_prefill(h0, layers, dims, halt_layer, mode="prune", select="topk",
                 keep=0.5, threshold=None, relative=False, keep_first=0,
                 keep_last=0, forced_idx=None, monitor_layers=1, return_kv=False):
    """Single-shot DASH prefill ([DASH blog] §2.3, §3.1; [DASH news]).

    Layers 0..halt_layer run on all T tokens (R6, R7).  After the halting
    layer, Δ is scored from its attention output U and the active set S* is
    chosen once; every later layer reuses it.

    mode 'prune': later layers run on the gathered rows only, each keeping its
      original position (R13).  Returns hidden [K, d].
    mode 'halt': halted rows keep the halting layer's output forever; their
      K/V, recomputed per layer from that frozen state (R12), stay visible to
      the active queries, which attend causally by original position.
      Returns hidden [T, d].

    monitor_layers = W > 1 takes Δ at the W consecutive layers ending at the
    halting layer and keeps their elementwise maximum ([DASH news]
    "层间更新动态监测": a token is stable when its update stays below the
    threshold over several consecutive layers; with threshold selection it
    halts iff Δ_l < threshold in every monitored layer).

    forced_idx, when given, replaces the selection (teacher forcing in tests).
    Returns a dict with hidden, idx, delta, halt_out (halting layer output)
    and halt_in (its input).  With return_kv, "kv" holds per layer the tuple
    (k, v, pos) of the keys/values that layer's attention read, in position
    order: the KV cache the prefill leaves for generation (R17).  In prune
    mode the layers after the halting layer hold the active rows only.
    """
    h = np.asarray(h0, dtype=np.float64)
    T = len(h)
    pos = np.arange(T)
    window = max(1, monitor_layers)
    if window > halt_layer + 1:
        raise OracleError("monitor window longer than the layers before halting")
    delta = None
    kv = [] if return_kv else None

    def block(h_q, q_pos, h_kv, kv_pos, w):
        k, v = layer_kv(h_kv, kv_pos, w, dims)
        if kv is not None:
            kv.append((k, v, np.asarray(kv_pos, dtype=np.int64)))
        return block_with_kv(h_q, q_pos, k, v, kv_pos, w, dims)

    for l in range(halt_layer + 1):
        h_in = h
        h, u = block(h, pos, h, pos, layers[l])
        if l > halt_layer - window:
            d_l = delta_scores(u, h_in, relative)
            delta = d_l if delta is None else np.maximum(delta, d_l)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, dtype=np.int64)
    elif select == "topk":
        idx = select_topk(delta, keep, keep_first, keep_last)
    elif select == "threshold":
        idx = select_threshold(delta, threshold, keep_first, keep_last)
    else:
        raise OracleError(f"unknown select {select!r}")
    halt_out = h
    if mode == "prune":
        hc = gather_rows(h, idx)
        for l in range(halt_layer + 1, len(layers)):
            hc, _ = block(hc, idx, hc, idx, layers[l])
        hidden = hc
    elif mode == "halt":
        hf = np.array(h, copy=True)
        for l in range(halt_layer + 1, len(layers)):
            new_rows, _ = block(hf[idx], idx, hf, pos, layers[l])
            hf[idx] = new_rows
        hidden = hf
    else:
        raise OracleError(f"unknown mode {mode!r}")
    out = {"hidden": hidden, "idx": idx, "delta": delta,
           "halt_out": halt_out, "halt_in": h_in}
    if kv is not None:
        out["kv"] = kv
    return out


def dash_prefill_varlen(h0, cu_seqlens, layers, dims, halt_layer, mode="prune", forced_idx=None, **kw):
    """A batch of independent sequences ([DASH blog] §5.1: every sample takes
    its own decision; gather/scatter must not mix samples).

    Sequence s is rows [cu[s], cu[s+1]) of h0.  The result is, by definition,
    the single-sequence prefill applied to each sequence on its own (RoPE
    positions from 0, attention within the sequence, its own selection),
    concatenated in order; idx holds absolute row numbers.  forced_idx, when
    given, is a global ascending index list split by sequence.
    """
    cu = [int(x) for x in cu_seqlens]
    h0 = np.asarray(h0, dtype=np.float64)
    hidden, idx, delta, counts, kvs = [], [], [], [], []
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        f = None
        if forced_idx is not None:
            g = np.asarray(forced_idx)
            f = g[(g >= a) & (g < b)] - a
        if b == a:
            counts.append(0)
            kvs.append(None)
            continue
        r = dash_prefill(h0[a:b], layers, dims, halt_layer, mode, forced_idx=f, **kw)
        kvs.append(r.get("kv"))
        hidden.append(r["hidden"])
        idx.append(r["idx"] + a)
        delta.append(r["delta"])
        counts.append(len(r["idx"]))
    d = h0.shape[1]
    out = {"hidden": np.concatenate(hidden) if hidden else np.zeros((0, d)),
           "idx": np.concatenate(idx).astype(np.int64) if idx else np.zeros(0, np.int64),
           "delta": np.concatenate(delta) if delta else np.zeros(0), "counts": counts}
    if kw.get("return_kv"):
        out["kv"] = kvs  # per sequence (positions within the sequence), None if empty
    return out


# ------------------------------------------------------------------- decode

def dash_decode(x, pos, kv, layers, dims):
    """Generation after a DASH prefill ([DASH blog] §3.1, generation stage, and
    §5.1 on the KV cache): no pruning is applied to generated tokens, but in
    every layer after the halting layer the cache holds only the active
    tokens, so the new tokens attend to fewer keys.

    x: [n, d] hidden states of n new tokens of one sequence at positions pos
    (R18: the original numbering continues, e.g. T for the first generated
    token).  kv: per layer (k, v, pos) as dash_prefill(return_kv=True)
    returns it.  Every layer runs on the new rows; they attend to the cached
    rows and causally to each other.  Returns (hidden [n, d], kv with the new
    rows appended).
    """
    h = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.int64)
    new_kv = []
    for w, (kc, vc, pc) in zip(layers, kv):
        kn, vn = layer_kv(h, pos, w, dims)
        k = np.concatenate([kc, kn])
        v = np.concatenate([vc, vn])
        p = np.concatenate([pc, pos])
        h, _ = block_with_kv(h, pos, k, v, p, w, dims)
        new_kv.append((k, v, p))
    return h, new_kv
