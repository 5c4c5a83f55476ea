"""Algorithmic work of the DASH prefill path (FLOPs and HBM bytes).

Counting rules: a linear layer costs 2 FLOPs per weight per token; causal
attention costs 4*hq*hd FLOPs per visible (query, key) pair (QK^T and PV);
HBM-bound kernels count the bytes they must read and write once.
"""


def linear_flops_per_token(dims):
    d, hd, F = dims.d_model, dims.head_dim, dims.ffn_dim
    qd, kvd = dims.n_heads * hd, dims.n_kv_heads * hd
    return 2 * d * (qd + 2 * kvd) + 2 * qd * d + 2 * d * 2 * F + 2 * F * d


def attn_flops(dims, pairs):
    return 4 * dims.n_heads * dims.head_dim * pairs


def causal_pairs(n):
    return n * (n + 1) // 2


def prefill_flops(dims, T, halt_layer=None, K=None, mode="dense", active_idx=None):
    """Total algorithmic FLOPs of one prefill.

    dense: every layer on T tokens.  prune: layers 0..halt_layer on T, later
    layers on K tokens with causal attention among them.  halt: later layers
    run K queries against all visible keys (sum of active positions + 1; K/T
    of the causal pairs when the positions are not given, as for evenly
    spread active rows) and recompute the K/V projections of the T-K halted
    rows.
    """
    lin = linear_flops_per_token(dims)
    full = T * lin + attn_flops(dims, causal_pairs(T))
    L = dims.n_layers
    if mode == "dense" or halt_layer is None:
        return L * full
    n_full = halt_layer + 1
    n_late = L - n_full
    if mode == "prune":
        late = K * lin + attn_flops(dims, causal_pairs(K))
    else:
        pairs = int(sum(int(i) + 1 for i in active_idx)) if active_idx is not None else causal_pairs(T) * K // T
        kvd = dims.n_kv_heads * dims.head_dim
        late = K * lin + attn_flops(dims, pairs) + (T - K) * 2 * dims.d_model * 2 * kvd
    return n_full * full + n_late * late


def varlen_prefill_flops(dims, cu, halt_layer=None, counts=None, mode="dense", active_idx=None):
    """prefill_flops summed over the independent sequences [cu[s], cu[s+1])."""
    total = 0
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        act = None
        if active_idx is not None:
            act = [int(i) - a for i in active_idx if a <= int(i) < b]
        total += prefill_flops(dims, b - a, halt_layer, None if counts is None else counts[s], mode, act)
    return total


def layer_weight_bytes(dims):
    """bf16 bytes of one decoder layer's weights (projections and norm gains)."""
    d, hd, F = dims.d_model, dims.head_dim, dims.ffn_dim
    qd, kvd = dims.n_heads * hd, dims.n_kv_heads * hd
    return 2 * (d * (qd + 2 * kvd) + qd * d + 2 * F * d + F * d + 2 * d)


def decode_step_bytes(dims, cache_lens):
    """HBM bytes one generation step must move: every layer's weights once,
    plus, per sequence and layer, the cached keys/values it attends over
    (cache_lens[s][l] rows after the append) and the appended row."""
    kvd = dims.n_kv_heads * dims.head_dim
    kv = sum(sum(lens) for lens in cache_lens) * kvd * 2 * 2
    return dims.n_layers * layer_weight_bytes(dims) + kv


def launch_work(rec, dims, pairs_by_rows=None):
    """(unit, amount) of algorithmic work for one timed launch record.  Attention
    launches whose visible pairs the library cannot count on the host (query
    positions or per-sequence key starts) record k = -1; pairs_by_rows maps their
    query-row count to the pairs of this run."""
    kind, m, n, k = rec["kind"], rec["m"], rec["n"], rec["k"]
    if kind.startswith("gemm"):
        return "flop", 2 * m * n * k
    if kind == "attention":
        pairs = k if k >= 0 else (pairs_by_rows or {}).get(m, 0)
        return "flop", attn_flops(dims, pairs)
    if kind == "rmsnorm":
        return "byte", 2 * m * n * 2
    if kind in ("gather", "scatter"):
        return "byte", 2 * m * n * 2
    if kind == "score":
        return "byte", m * 4 * (2 * n + 1) if n < 1024 else m * n * 2 * (1 + k) + 4 * m
    if kind == "select":
        return "byte", m * 4 + m * 4
    if kind == "rope_table":
        return "byte", m * n * 8
    if kind.startswith("gemv"):          # weights [n, k] once, m input rows, m output rows
        return "byte", 2 * (n * k + m * k + m * n)
    if kind == "decode_attention":       # n cached rows (summed over sequences), K and V
        return "byte", n * dims.n_kv_heads * dims.head_dim * 2 * 2
    if kind == "kv_store":               # m rows of K and V read and written
        return "byte", m * n * 2 * 2 * 2
    return "byte", 0
