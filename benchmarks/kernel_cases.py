"""Runs one kernel of the DASH prefill path at a chosen shape (for timing and
for ncu captures of a single kernel on a small case).

    python benchmarks/kernel_cases.py attention --T 8192
    python benchmarks/kernel_cases.py linear --M 4096 --N 37888 --K 3584
    python benchmarks/kernel_cases.py layer --T 4096
    python benchmarks/kernel_cases.py select --T 32768
    python benchmarks/kernel_cases.py decode --T 32768 --M 1
    python benchmarks/kernel_cases.py decode_attention --T 32768 --M 1
    python benchmarks/kernel_cases.py rows --T 32768

Shapes default to the Qwen2.5-7B-shaped stack (28 q / 4 kv heads, hd 128,
d 3584, FFN 18944).  Prints one JSON line with the mean CUDA-event time.
"""
import argparse
import json
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from long_context_prefill_tcgen05_b200 import build, costs, dash, inputs  # noqa: E402


def _time(fn, iters, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["attention", "linear", "layer", "select", "score", "gather", "decode",
                                     "decode_attention", "rows"])
    ap.add_argument("--T", type=int, default=8192)
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=37888)
    ap.add_argument("--K", type=int, default=3584)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--layers", type=int, default=1, help="decode: layers of the stack")
    args = ap.parse_args()
    build.build()
    dims = inputs.QWEN7B
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    rnd = lambda *s: torch.randn(*s, generator=g, device=dev).to(torch.bfloat16)
    out = {"case": args.case}
    if args.case == "attention":
        T, hq, hkv, hd = args.T, dims.n_heads, dims.n_kv_heads, dims.head_dim
        Q, K, V = rnd(T, hq * hd), rnd(T, hkv * hd), rnd(T, hkv * hd)
        O = torch.empty_like(Q)
        ms = _time(lambda: dash.attention(Q, K, V, hq, hkv, hd, out=O), args.iters, args.warmup)
        fl = costs.attn_flops(dims, costs.causal_pairs(T))
        out.update(T=T, ms=ms, tflops=fl / ms / 1e9)
    elif args.case == "linear":
        A, W = rnd(args.M, args.K), rnd(args.N, args.K) * 0.02
        Y = torch.empty(args.M, args.N, dtype=torch.bfloat16, device=dev)
        ms = _time(lambda: dash.linear(A, W, out=Y), args.iters, args.warmup)
        out.update(M=args.M, N=args.N, K=args.K, ms=ms, tflops=2 * args.M * args.N * args.K / ms / 1e9)
    elif args.case == "layer":
        stack = dash.Stack(dims, inputs.make_layers(dims, seed=0, device=dev, n_layers=1))
        h0 = rnd(args.T, dims.d_model)
        H = torch.empty_like(h0)
        delta = torch.empty(args.T, device=dev)

        def run():
            H.copy_(h0)
            dash.layer_forward(stack, 0, H, delta=delta)
        ms = _time(run, args.iters, args.warmup)
        fl = args.T * costs.linear_flops_per_token(dims) + costs.attn_flops(dims, costs.causal_pairs(args.T))
        out.update(T=args.T, ms=ms, tflops=fl / ms / 1e9)
    elif args.case == "select":
        s = torch.rand(args.T, generator=g, device=dev)
        ms = _time(lambda: dash.select(s, "topk", 0.5), args.iters, args.warmup)
        out.update(T=args.T, ms=ms)
    elif args.case == "score":
        U = rnd(args.T, dims.d_model)
        d = torch.empty(args.T, device=dev)
        ms = _time(lambda: dash.score(U, out=d), args.iters, args.warmup)
        out.update(T=args.T, ms=ms, gbs=args.T * dims.d_model * 2 / ms / 1e6)
    elif args.case == "gather":
        X = rnd(args.T, dims.d_model)
        idx = torch.sort(torch.randperm(args.T, generator=g, device=dev)[:args.T // 2]).values.int()
        ms = _time(lambda: dash.compact(X, idx), args.iters, args.warmup)
        out.update(T=args.T, ms=ms, gbs=2 * (args.T // 2) * dims.d_model * 2 / ms / 1e6)
    elif args.case == "rows":
        # RMSNorm, score (absolute and relative), gather and scatter of T/2 rows, and
        # top-k select, each launch timed alone with L2 flushed before it (cold HBM)
        T, d = args.T, dims.d_model
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

        def cold(fn, n=20):
            ts = []
            for i in range(n + 3):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                if i >= 3:
                    ts.append(e0.elapsed_time(e1))
            return sorted(ts)[len(ts) // 2]
        U, H = rnd(T, d), rnd(T, d)
        delta = torch.empty(T, device=dev)
        K = T // 2
        idx = torch.sort(torch.randperm(T, generator=g, device=dev)[:K]).values.int()
        Y = dash.compact(U, idx)
        s = torch.rand(T, generator=g, device=dev)
        sel_idx = torch.empty(T, dtype=torch.int32, device=dev)
        count = torch.empty(1, dtype=torch.int32, device=dev)
        L = dash.lib()
        sel_ws = torch.empty(L.dash_select_workspace_size(T), dtype=torch.uint8, device=dev)
        gain = (1 + 0.1 * torch.randn(d, generator=g, device=dev)).bfloat16()
        Yn = torch.empty_like(H)
        ms = {
            "rmsnorm": cold(lambda: dash._check(L.dash_rmsnorm(dash._p(H), T, d, dash._p(gain), 1e-6, dash._p(Yn), None),
                                                "dash_rmsnorm")),
            "score": cold(lambda: dash.score(U, out=delta)),
            "score_relative": cold(lambda: dash.score(U, H, relative=True, out=delta)),
            "gather": cold(lambda: dash.compact(U, idx)),
            "scatter": cold(lambda: dash.scatter(Y, idx, H)),
            "select": cold(lambda: L.dash_select(dash._p(s), T, dash.SELECTS["topk"], 0.5, 0.0, 0, 0,
                                                 dash._p(sel_idx), None, dash._p(count), dash._p(sel_ws),
                                                 sel_ws.numel(), None)),
        }
        nbytes = {"rmsnorm": 2 * T * d * 2, "score": T * d * 2, "score_relative": 2 * T * d * 2, "gather": 2 * K * d * 2,
                  "scatter": 2 * K * d * 2, "select": T * 4 + K * 4}
        out.update(T=T, d=d, K=K, us={k: round(v * 1e3, 1) for k, v in ms.items()},
                   gbs={k: round(nbytes[k] / ms[k] / 1e6) for k in ms})
        dash.check_device()
    elif args.case in ("decode", "decode_attention"):
        # one generation step of a stack of --layers layers (or one layer's
        # attention alone) for M sequences, each with a cache of T random rows
        n, T, nl = args.M, args.T, args.layers
        hq, hkv, hd = dims.n_heads, dims.n_kv_heads, dims.head_dim
        stack = dash.Stack(dims, inputs.make_layers(dims, seed=0, device=dev, n_layers=nl))
        cap = T + args.iters + args.warmup + 1
        cache = dash.KVCache(stack, n, cap, device=dev)
        for i in range(n * nl):
            cache.k[i][:T] = rnd(T, hkv * hd)
            cache.v[i][:T] = rnd(T, hkv * hd)
            cache.desc[i].len = T
        if args.case == "decode":
            X = rnd(n, dims.d_model)
            step = [T]

            def run():
                dash.decode_step(stack, X, [step[0]] * n, cache)
                step[0] += 1
            ms = _time(run, args.iters, args.warmup)
            by = nl * (costs.layer_weight_bytes(dims) + n * (T + 1) * hkv * hd * 2 * 2)
        else:
            Q = rnd(n, hq * hd)
            O = torch.empty_like(Q)
            kv = [(cache.k[i * nl][:T], cache.v[i * nl][:T]) for i in range(n)]
            ms = _time(lambda: dash.decode_attention(Q, kv, hq, hkv, hd, out=O), args.iters, args.warmup)
            by = n * T * hkv * hd * 2 * 2
        out.update(T=T, n=n, ms=ms, gbs=by / ms / 1e6)
    dash.check_device()
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
