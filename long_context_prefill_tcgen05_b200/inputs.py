"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module draws random numbers and arranges them in the layouts the
workloads need.  It holds none of the method's arithmetic (no norms, no
attention, no selection), so feeding both sides from it couples nothing but
their inputs.

Workloads (shapes follow the long-context text-prefill setting of the DASH
pages: a Qwen2.5-7B-class stack, 32K-128K tokens; weights are random-init
because no trained checkpoint is available):

  tiny      4 layers, d=256, 4 q / 2 kv heads, hd=64, FFN 704, θ=1e4, T=512
  qwen7b    28 layers, d=3584, 28 q / 4 kv heads, hd=128, FFN 18944, θ=1e6
  llama8b   32 layers, d=4096, 32 q / 8 kv heads, hd=128, FFN 14336, θ=5e5

Weights are bf16 N(0, 0.02) drawn layer by layer in the fixed order
wq, wk, wv, wo, wg, wu, wd; norm gains are 1.  Hidden inputs are bf16 N(0, 1).
"""
from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class ModelDims:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_dim: int
    rope_theta: float
    rms_eps: float = 1e-6

    def as_dict(self):
        return asdict(self)

    @property
    def qkv_dim(self):
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim


TINY = ModelDims(4, 256, 4, 2, 64, 704, 1e4)
QWEN7B = ModelDims(28, 3584, 28, 4, 128, 18944, 1e6)
LLAMA8B = ModelDims(32, 4096, 32, 8, 128, 14336, 5e5)


def _randn(shape, gen, device, std=1.0):
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def make_layers(dims: ModelDims, seed: int = 0, device="cpu", n_layers=None):
    """Per-layer weight dicts of bf16 tensors (row-major [out, in] like nn.Linear).

    Keys: attn_norm [d], wq [hq*hd, d], wk [hkv*hd, d], wv [hkv*hd, d],
    wo [d, hq*hd], ffn_norm [d], wg [F, d], wu [F, d], wd [d, F].
    """
    gen = torch.Generator(device=device).manual_seed(seed)
    d, hd, F = dims.d_model, dims.head_dim, dims.ffn_dim
    layers = []
    for _ in range(dims.n_layers if n_layers is None else n_layers):
        w = {}
        w["wq"] = _randn((dims.n_heads * hd, d), gen, device, 0.02)
        w["wk"] = _randn((dims.n_kv_heads * hd, d), gen, device, 0.02)
        w["wv"] = _randn((dims.n_kv_heads * hd, d), gen, device, 0.02)
        w["wo"] = _randn((d, dims.n_heads * hd), gen, device, 0.02)
        w["wg"] = _randn((F, d), gen, device, 0.02)
        w["wu"] = _randn((F, d), gen, device, 0.02)
        w["wd"] = _randn((d, F), gen, device, 0.02)
        w["attn_norm"] = torch.ones(d, dtype=torch.bfloat16, device=device)
        w["ffn_norm"] = torch.ones(d, dtype=torch.bfloat16, device=device)
        layers.append(w)
    return layers


def make_hidden(T: int, d: int, seed: int = 0, device="cpu", span_rows=0, span_len=64,
                span_scale=4.0):
    """Input hidden states H0 [T, d] bf16 N(0, 1).

    With span_rows > 0, span_rows // span_len non-overlapping spans of span_len
    consecutive rows (starts drawn on a span_len-aligned grid) are scaled by
    span_scale -- the "x4 rows in contiguous spans" structure of the
    score/select and 128K workloads.
    Returns (H0, scaled_row_mask).
    """
    gen = torch.Generator(device=device).manual_seed(seed)
    h = torch.randn(T, d, generator=gen, device=device, dtype=torch.float32)
    mask = torch.zeros(T, dtype=torch.bool, device=device)
    n_spans = span_rows // span_len
    if n_spans:
        slots = T // span_len
        pick = torch.randperm(slots, generator=gen, device=device)[:n_spans]
        for s in pick.tolist():
            mask[s * span_len:(s + 1) * span_len] = True
        h[mask] *= span_scale
    return h.to(torch.bfloat16), mask


def make_score_bench_inputs(T=32768, d=3584, seed=1, device="cpu"):
    """Score+select microbenchmark inputs: U and H bf16 [T, d] N(0,1), with 10%
    of U's rows (51 spans of 64 rows = 3264 rows) scaled by 4."""
    u, mask = make_hidden(T, d, seed, device, span_rows=(T // 10) // 64 * 64, span_len=64)
    gen = torch.Generator(device=device).manual_seed(seed + 1000)
    h = torch.randn(T, d, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return u, h, mask


def make_varlen_hidden(n_seq=4, seq_len=16384, text_len=2048, d=4096, n_centres=256,
                       seed=0, device="cpu"):
    """Varlen batch: each sequence = text_len N(0,1) rows, then rows drawn as
    centre[c] + N(0, 0.1) with c uniform over n_centres N(0,1) centres."""
    gen = torch.Generator(device=device).manual_seed(seed)
    seqs = []
    for _ in range(n_seq):
        text = torch.randn(text_len, d, generator=gen, device=device)
        centres = torch.randn(n_centres, d, generator=gen, device=device)
        c = torch.randint(0, n_centres, (seq_len - text_len,), generator=gen, device=device)
        vis = centres[c] + 0.1 * torch.randn(seq_len - text_len, d, generator=gen, device=device)
        seqs.append(torch.cat([text, vis]))
    h = torch.cat(seqs).to(torch.bfloat16)
    cu = torch.arange(0, (n_seq + 1) * seq_len, seq_len, dtype=torch.int32)
    return h, cu


def adversarial_scores(kind: str, T: int, seed: int = 0):
    """fp32 score vectors that stress selection: ties, signed zeros, denormals."""
    gen = torch.Generator().manual_seed(seed)
    if kind == "random":
        return torch.rand(T, generator=gen)
    if kind == "all_equal":
        return torch.full((T,), 0.5)
    if kind == "few_values":      # heavy ties everywhere, including at the cut
        return torch.randint(0, 4, (T,), generator=gen).float() * 0.25
    if kind == "signed_zero":     # +0 / -0 mixed with a few positives
        x = torch.zeros(T)
        x[torch.rand(T, generator=gen) < 0.5] = -0.0
        x[torch.randint(0, T, (max(1, T // 16),), generator=gen)] = 1.0
        return x
    if kind == "denormal":
        m = torch.randint(1, 1 << 10, (T,), generator=gen, dtype=torch.int32)
        return m.view(torch.float32)  # bit patterns of positive subnormals
    if kind == "negative":
        return torch.randn(T, generator=gen)
    if kind == "spiky":           # long flat run with rare large values
        x = torch.full((T,), 1e-3)
        x[torch.randint(0, T, (max(1, T // 100),), generator=gen)] = 10.0
        return x
    if kind == "narrow":          # distinct values sharing their top key bits (one bucket holds them all)
        return 1.0 + torch.rand(T, generator=gen) * 1e-3
    raise ValueError(kind)
