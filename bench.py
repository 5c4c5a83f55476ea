#!/usr/bin/env python
"""DASH long-context prefill benchmark on B200: prefill tokens/s, halted vs dense.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qwen7b-32k]
                    [--mode prune|halt] [--impl ours|reference]

One step = one full prefill (all layers, selection, compaction) of one
synthetic sequence through libdash's C ABI, inputs resident in HBM.  The
headline `value` is the halted (DASH) prefill; the same kernels without
halting give the dense figure.  With N > 1 (torchrun), every rank runs an
independent replica (the path has no data-parallel exchange) and the time is
the max over ranks.  Prints ONE JSON line on rank 0.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_prefill_tcgen05_b200 import costs, inputs  # noqa: E402

WORKLOADS = {
    "qwen7b-32k": dict(dims=inputs.QWEN7B, T=32768, halt_layer=11, keep=0.5, select="topk", relative=False,
                       span_rows=0, span_len=64, mode="prune",
                       name="Qwen2.5-7B-shaped stack (28 layers, d=3584, 28q/4kv, hd=128, FFN 18944), "
                            "T=32768, halt at layer 11, keep 0.5"),
    # threshold = the relative delta at rank floor(0.3 T) of a calibration prefill on the
    # same input, then frozen (the timed run is a pure threshold run)
    "qwen7b-128k": dict(dims=inputs.QWEN7B, T=131072, halt_layer=11, keep=0.3, select="threshold", relative=True,
                        span_rows=6528, span_len=128, mode="halt", calibrate=True,
                        name="Qwen2.5-7B-shaped stack, T=131072, halt at layer 11, relative-delta threshold "
                             "calibrated to keep 30%, halt mode"),
    "llama8b-varlen": dict(dims=inputs.LLAMA8B, T=65536, nseq=4, halt_layer=13, keep=0.4, select="topk",
                           relative=False, span_rows=0, span_len=64, mode="prune", varlen=True,
                           name="Llama-3.1-8B-shaped stack (32 layers, d=4096, 32q/8kv, hd=128, FFN 14336), varlen "
                                "batch 4 x 16384 (2048 text + 14336 clustered rows each), halt at layer 13, keep 0.4"),
    "tiny": dict(dims=inputs.TINY, T=512, halt_layer=2, keep=0.5, select="topk", relative=False, span_rows=0,
                 span_len=64, mode="prune", name="tiny decoder stack (4 layers, d=256, 4q/2kv, hd=64, FFN 704), T=512"),
}
METRIC = "prefill tokens/s @T=32K/128K, halted vs dense, and % of B200 roofline"


def recorded_traffic(kind, recs):
    """DRAM bytes per launch of `kind` from the committed ncu record, scaled by rows to
    the launches of this run; None when the kernel source changed since the capture."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kind)
        src = os.path.join(ROOT, "long_context_prefill_tcgen05_b200", "csrc", f"{kind}.cuh")
        with open(src, "rb") as f:
            if rec is None or hashlib.sha256(f.read()).hexdigest() != rec["src_sha256"]:
                return None
    except (OSError, ValueError, KeyError):
        return None
    launches = [r for r in recs if r["kind"] == kind]
    return sum(rec["bytes_per_launch"] * r["m"] / rec["rows"] for r in launches) / max(1, len(launches))


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------ distributed
def dist_env():
    """(world, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup(backend=None, timeout_s=600):
    """One process per GPU: NCCL when CUDA is present, else gloo (CPU tests of the
    multi-rank host logic).  The replicas exchange only timing results."""
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The maximum of x over the ranks (multi-GPU times are the slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# -------------------------------------------------------------- CPU side
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        if blas:
            return int(max(blas))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample_time(dims, layer_np, T_s, seed=0):
    """Seconds for the oracle to run one decoder block of the stack on T_s tokens."""
    import numpy as np
    import oracle as O
    h = inputs.make_hidden(T_s, dims.d_model, seed=seed)[0].double().numpy()
    pos = np.arange(T_s)
    t0 = time.perf_counter()
    O.decoder_block(h, pos, h, pos, layer_np, dims.as_dict())
    return time.perf_counter() - t0


def cpu_layer_np(dims):
    layer = inputs.make_layers(dims, seed=0, device="cpu", n_layers=1)[0]
    return {k: v.double().numpy() for k, v in layer.items()}


def cpu_sample_tokens(dims, T):
    """Tokens of the bounded CPU sample: one decoder block on 2048 tokens for
    the 7B/8B-shaped stacks (a few seconds of fp64 work on 16 cores), the
    whole sequence for the tiny stack."""
    return min(T, 2048)


def cpu_rate(dims, T, target_flops, t, T_s):
    """tokens/s of the whole workload from one sample: T_s tokens through one
    block in t seconds, extrapolated by algorithmic FLOPs."""
    f_s = T_s * costs.linear_flops_per_token(dims) + costs.attn_flops(dims, costs.causal_pairs(T_s))
    return T / (t * target_flops / f_s), f_s


def cpu_baseline(dims, T, target_flops, samples=3):
    """The oracle timed on host cores on a bounded sample of the workload --
    the same sample the reference arm times per step -- median of `samples`."""
    layer_np = cpu_layer_np(dims)
    T_s = cpu_sample_tokens(dims, T)
    ts = [oracle_sample_time(dims, layer_np, T_s) for _ in range(samples)]
    t = statistics.median(ts)
    value, f_s = cpu_rate(dims, T, target_flops, t, T_s)
    return {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"one decoder block of the same stack on {T_s} tokens ({f_s / 1e9:.0f} GFLOP fp64, "
                      f"median {t:.2f} s of {samples}), extrapolated by algorithmic FLOPs to the full prefill",
            "sample_seconds": t}


# ------------------------------------------------------------ reference
def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores: each step is the bounded
    sample cpu_baseline takes (one block on the same tokens), extrapolated
    the same way; rank 0 alone runs it."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    dims, T = wl["dims"], wl["T"]
    mode = args.mode or wl["mode"]
    K = math.floor(wl["keep"] * T)
    target = costs.prefill_flops(dims, T, wl["halt_layer"], K, mode)
    layer_np = cpu_layer_np(dims)
    T_s = cpu_sample_tokens(dims, T)
    for _ in range(args.warmup):
        oracle_sample_time(dims, layer_np, T_s)
    ts = [oracle_sample_time(dims, layer_np, T_s) for _ in range(args.steps)]
    t = sum(ts) / len(ts)
    value, f_s = cpu_rate(dims, T, target, t, T_s)
    cb = {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
          "sample": f"each step: one decoder block of the same stack on {T_s} tokens ({f_s / 1e9:.0f} GFLOP fp64, "
                    f"mean {t:.2f} s), extrapolated by algorithmic FLOPs to the full halted prefill"}
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
                      "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": t * target / f_s * 1e3, "higher_is_better": True, "scaling": "weak",
                      "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                      "config": {"workload": wl["name"], "seq_len": T, "halt_layer": wl["halt_layer"],
                                 "keep": wl["keep"], "mode": mode},
                      "cpu_baseline": cb,
                      "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)


# --------------------------------------------------------------- decode
def decode_leg(dash, stack, dims, wl, h0, cu, cfg_cache, cfg_dense, dev, peaks, block=8, rounds=5, warmup=3):
    """Generation after the prefill: ms per step (one new token per sequence)
    on the cache a DASH prefill leaves (prune mode: later layers hold the
    active tokens only) against the dense prefill's cache.  Both caches are
    resident; timed blocks of `block` steps alternate between them and the
    median block is reported."""
    nseq = len(cu) - 1 if cu else 1
    T_max = max(b - a for a, b in zip(cu[:-1], cu[1:])) if cu else h0.shape[0]
    total = warmup + rounds * block + block  # + one block with per-kernel events
    g = torch.Generator(device=dev).manual_seed(99)
    starts = [cu[s + 1] - cu[s] for s in range(nseq)] if cu else [h0.shape[0]]
    legs = {}
    for name, c in (("dash_cache", cfg_cache), ("dense_cache", cfg_dense)):
        cache = dash.KVCache(stack, nseq, T_max + total, device=dev)
        H = h0.clone()
        if cu:
            dash.prefill_varlen_kv(stack, H, cu, c, cache)
        else:
            dash.prefill_kv(stack, H, c, cache)
        del H
        xs = torch.randn(total, nseq, dims.d_model, generator=g, device=dev).to(torch.bfloat16)
        legs[name] = {"cache": cache, "xs": xs, "j": 0, "ms": [], "rows": cache.lens(0)}

    def run(leg, k):
        for _ in range(k):
            j = leg["j"]
            dash.decode_step(stack, leg["xs"][j], [p + j for p in starts], leg["cache"])
            leg["j"] += 1

    for leg in legs.values():
        run(leg, warmup)
    torch.cuda.synchronize()
    for _ in range(rounds):
        for leg in legs.values():
            base = [leg["cache"].lens(s) for s in range(nseq)]
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run(leg, block)
            e1.record()
            torch.cuda.synchronize()
            leg["ms"].append(e0.elapsed_time(e1) / block)
            leg.setdefault("bytes", []).append(sum(
                costs.decode_step_bytes(dims, [[b + 1 + j for b in base[s]] for s in range(nseq)])
                for j in range(block)) / block)
    out = {}
    for name, leg in legs.items():
        dash.timing_start()
        run(leg, block)
        torch.cuda.synchronize()
        recs = dash.timing_stop()
        per = {}
        for r in recs:
            unit, amount = costs.launch_work(r, dims)
            q = per.setdefault(r["kind"], {"ms": 0.0, "bytes": 0, "launches": 0})
            q["ms"] += r["ms"]
            q["bytes"] += amount
            q["launches"] += r.get("launches", 1)
        dom = max(per, key=lambda k: per[k]["ms"])
        gbs = per[dom]["bytes"] / (per[dom]["ms"] / 1e3) / 1e9
        ms = statistics.median(leg["ms"])
        step_bytes = statistics.median(leg["bytes"])
        out[name] = {"ms_per_step": ms, "ms_blocks": leg["ms"], "tokens_per_s": nseq / (ms / 1e3),
                     "cached_rows_per_layer": leg["rows"],
                     "step_gb": step_bytes / 1e9, "step_gbs": step_bytes / (ms / 1e3) / 1e9,
                     "step_frac_of_hbm": step_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "gpu_launches_per_step": sum(r.get("launches", 1) for r in recs) // block,
                     "kernels": {k: {"ms_per_step": v["ms"] / block, "launches_per_step": v["launches"] // block,
                                     "gbs": v["bytes"] / (v["ms"] / 1e3) / 1e9 if v["ms"] else 0.0}
                                 for k, v in sorted(per.items(), key=lambda kv: -kv[1]["ms"])},
                     "roofline": {"bound": "hbm", "kernel": dom, "achieved": gbs, "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                                  "note": "per-kernel times from CUDA events around each launch"}}
    del legs
    torch.cuda.empty_cache()
    out["speedup_vs_dense_cache"] = out["dense_cache"]["ms_per_step"] / out["dash_cache"]["ms_per_step"]
    out["sequences"] = nseq
    out["timing"] = f"median of {rounds} blocks of {block} steps per cache, blocks alternating, after {warmup} warm-up steps"
    return out


# ------------------------------------------------------------ prefill legs
class Prefill:
    """One workload's buffers and its prefill step on a stack (inputs resident)."""

    def __init__(self, dash, stack, h0, cu, world):
        self.dash, self.stack, self.h0, self.cu, self.world = dash, stack, h0, cu, world
        T = h0.shape[0]
        self.H = torch.empty_like(h0)
        self.idx = torch.empty(T, dtype=torch.int32, device=h0.device)
        self.delta = torch.empty(T, dtype=torch.float32, device=h0.device)

    def run(self, c, H=None, stream=None):
        H = self.H if H is None else H
        if self.cu:
            return self.dash.prefill_varlen(self.stack, H, self.cu, c, idx_out=self.idx, delta_out=self.delta,
                                            stream=stream)[0]
        return self.dash.prefill(self.stack, H, c, idx_out=self.idx, delta_out=self.delta, stream=stream)

    def step(self, c):
        self.H.copy_(self.h0)
        return self.run(c)

    def timed(self, c, k, record=False):
        """ms per step over k steps (max over ranks), the last K, and the launch
        records when record is set (CUDA events around every launch)."""
        torch.cuda.synchronize()
        barrier(self.world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if record:
            self.dash.timing_start()
        e0.record()
        K = None
        for _ in range(k):
            K = self.step(c)
        e1.record()
        torch.cuda.synchronize()
        recs = self.dash.timing_stop() if record else None
        barrier(self.world)
        return max_over_ranks(e0.elapsed_time(e1) / k, self.world), K, recs

    def calibrate_threshold(self, wl, mode):
        """The relative-Δ threshold that keeps ~wl['keep'] of the tokens: Δ at
        rank floor(keep T) of a top-k prefill on the same input, then frozen."""
        cal = self.dash.make_config(halt_layer=wl["halt_layer"], mode=mode, select="topk", keep=wl["keep"],
                                    relative=wl["relative"])
        self.step(cal)
        k = math.floor(wl["keep"] * self.h0.shape[0])
        return float(torch.sort(self.delta.cpu(), descending=True).values[k - 1])


def work_accounting(dims, T, cu, mode, halt_layer, K, active):
    """(halted FLOPs, visible pairs by attention query rows) of one prefill."""
    if cu:
        counts = [int(((active >= a) & (active < b)).sum()) for a, b in zip(cu[:-1], cu[1:])]
        flops = costs.varlen_prefill_flops(dims, cu, halt_layer, counts, mode, active)
        seq_of = lambda i: max(s for s in range(len(cu) - 1) if cu[s] <= i)
        pairs = {T: sum(costs.causal_pairs(b - a) for a, b in zip(cu[:-1], cu[1:]))}
        pairs[K] = (sum(costs.causal_pairs(k) for k in counts) if mode == "prune"
                    else int(sum(int(i) - cu[seq_of(int(i))] + 1 for i in active)))
    else:
        flops = costs.prefill_flops(dims, T, halt_layer, K, mode, active)
        pairs = {T: costs.causal_pairs(T), K: int(sum(int(i) + 1 for i in active))
                 if mode == "halt" else costs.causal_pairs(K)}
    return flops, pairs


def kernel_breakdown(recs, dims, pairs_by_rows, steps, peaks):
    """Per-kernel time and rate of `steps` instrumented steps, and the roofline
    of the dominant kernel (the kind with the most time)."""
    per = {}
    for r in recs:
        unit, amount = costs.launch_work(r, dims, pairs_by_rows)
        p = per.setdefault(r["kind"], {"launches": 0, "ms": 0.0, "unit": unit, "work": 0})
        p["launches"] += r.get("launches", 1)
        p["ms"] += r["ms"]
        p["work"] += amount
    total_ms = sum(p["ms"] for p in per.values())
    kernels = {}
    for kind, p in sorted(per.items(), key=lambda kv: -kv[1]["ms"]):
        rate = p["work"] / (p["ms"] / 1e3) if p["ms"] > 0 else 0.0
        kernels[kind] = {"launches_per_step": p["launches"] // steps, "ms_per_step": p["ms"] / steps,
                         "share": p["ms"] / total_ms if total_ms else 0.0,
                         ("tflops" if p["unit"] == "flop" else "gbs"): rate / 1e12 if p["unit"] == "flop"
                         else rate / 1e9}
    # GEMMs and attention split by the rows each launch processes (full-length
    # layers vs the compacted ones after the halting layer)
    by_rows = {}
    for r in recs:
        if r["kind"].startswith("gemm") or r["kind"] == "attention":
            unit, amount = costs.launch_work(r, dims, pairs_by_rows)
            q = by_rows.setdefault(f"{r['kind']}@{r['m']}", {"ms": 0.0, "work": 0, "launches": 0})
            q["ms"] += r["ms"]
            q["work"] += amount
            q["launches"] += r.get("launches", 1)
    for k, q in by_rows.items():
        kernels.setdefault("by_rows", {})[k] = {"launches_per_step": q["launches"] // steps,
                                                "tflops": q["work"] / (q["ms"] / 1e3) / 1e12 if q["ms"] else 0.0}
    dom_kind = max(per, key=lambda k: per[k]["ms"])
    dom = per[dom_kind]
    n_launch = sum(r.get("launches", 1) for r in recs)
    if dom["unit"] == "flop":
        achieved = dom["work"] / (dom["ms"] / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak}
    else:
        achieved = dom["work"] / (dom["ms"] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak}
    roof.update({"kernel": dom_kind, "traffic": recorded_traffic(dom_kind, recs),
                 "peak_source": f"{peaks['source']} ({'sustained bf16' if dom['unit'] == 'flop' else 'HBM copy'})"})
    return kernels, roof, n_launch // steps


def long_context_leg(dash, stack, dims, dev, peaks, world, rounds=2):
    """The T = 131072 workload on the same stack: halt mode with the relative-Δ
    threshold calibrated to keep ~30 %, against the dense prefill on the same
    kernels (single steps alternating), with its own kernel roofline."""
    wl = WORKLOADS["qwen7b-128k"]
    T = wl["T"]
    h0, _ = inputs.make_hidden(T, dims.d_model, seed=0, device=dev, span_rows=wl["span_rows"],
                               span_len=wl["span_len"])
    pf = Prefill(dash, stack, h0, None, world)
    thr = pf.calibrate_threshold(wl, wl["mode"])
    cfg = dash.make_config(halt_layer=wl["halt_layer"], mode=wl["mode"], select="threshold", threshold=thr,
                           relative=True)
    cfg_dense = dash.make_config(mode="dense")
    pf.step(cfg)
    pf.step(cfg_dense)
    legs = [(cfg, []), (cfg_dense, [])]
    for r in range(rounds):
        for c, times in (legs if r % 2 == 0 else legs[::-1]):
            times.append(pf.timed(c, 1)[0])
    ms_h, ms_d = (statistics.median(t) for _, t in legs)
    _, K, recs = pf.timed(cfg, 1, record=True)
    active = pf.idx[:K].cpu().numpy()
    flops, pairs = work_accounting(dims, T, None, wl["mode"], wl["halt_layer"], K, active)
    dense_flops = costs.prefill_flops(dims, T)
    kernels, roof, launches = kernel_breakdown(recs, dims, pairs, 1, peaks)
    dash.check_device()
    out = {"workload": wl["name"], "threshold": thr, "K": K, "kept": K / T,
           "value": world * T / (ms_h / 1e3), "unit": "tokens/s", "ms_per_step": ms_h,
           "dense": {"tokens_per_s": world * T / (ms_d / 1e3), "ms_per_step": ms_d,
                     "tflops": dense_flops / (ms_d / 1e3) / 1e12},
           "speedup_vs_dense": ms_d / ms_h, "flop_bound": dense_flops / flops,
           "halted_tflop_per_step": flops / 1e12, "step_tflops": flops / (ms_h / 1e3) / 1e12,
           "roofline": roof, "kernels": {k: v for k, v in list(kernels.items())[:6]},
           "gpu_launches_per_step": launches,
           "timing": f"median of {rounds} single steps per leg, halt / dense alternating; inputs larger than L2"}
    del pf, h0
    torch.cuda.empty_cache()
    return out


def fp16_leg(dash, wl, dims, h0, cu, cfg, pf16_of, pf_bf16, world, rounds=3):
    """The same workload with the model stored in fp16 (dash_dims.dtype =
    fp16: weights and every stored activation 16-bit fp16, fp32 accumulation),
    timed in single steps alternating with the bf16 path."""
    pf16 = pf16_of()
    pf16.step(cfg)
    legs = [(pf_bf16, []), (pf16, [])]
    for r in range(rounds):
        for p, times in (legs if r % 2 == 0 else legs[::-1]):
            times.append(p.timed(cfg, 1)[0])
    ms_b, ms_h = (statistics.median(t) for _, t in legs)
    dash.check_device()
    T = h0.shape[0]
    out = {"dtype": "f16", "value": world * T / (ms_h / 1e3), "unit": "tokens/s", "ms_per_step": ms_h,
           "bf16_ms_per_step": ms_b, "cost_vs_bf16": ms_h / ms_b,
           "timing": f"median of {rounds} single steps per format, alternating",
           "note": "fp16 storage holds the stated delta tolerance at the halting depth (tests/test_gpu_fp16.py)"}
    del pf16
    torch.cuda.empty_cache()
    return out


def score_select_leg(dash, dev, peaks, reps=20):
    """The score / select / compaction workload on its own: U, H bf16
    [32768, 3584] N(0,1), 10 % of U's rows x4 in 64-row spans (seed 1); Δ
    absolute and relative; top-k keep 0.5 and threshold = the median Δ
    (sorted int32 lists); gather of the K = 16384 kept rows.  Each launch is
    timed alone after a write of 256 MB (larger than L2), median of reps."""
    T, d = 32768, inputs.QWEN7B.d_model
    U, H, mask = inputs.make_score_bench_inputs(T, d, seed=1, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    L = dash.lib()
    delta = torch.empty(T, device=dev)
    delta_r = torch.empty(T, device=dev)
    idx = torch.empty(T, dtype=torch.int32, device=dev)
    count = torch.empty(1, dtype=torch.int32, device=dev)
    dash.score(U, out=delta)
    med = float(torch.median(delta).item())
    K = math.floor(0.5 * T)
    sel = dash.select(delta, "topk", 0.5)[0].clone()
    Y = torch.empty(K, d, dtype=torch.bfloat16, device=dev)

    def cold(fn):
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    sel_ws = torch.empty(L.dash_select_workspace_size(T), dtype=torch.uint8, device=dev)

    def select_call(kind, keep, thr):
        return lambda: L.dash_select(dash._p(delta), T, dash.SELECTS[kind], keep, thr, 0, 0, dash._p(idx), None,
                                     dash._p(count), dash._p(sel_ws), sel_ws.numel(), None)
    T2 = 131072  # the long-context length: selection over a 4x longer score vector
    g = torch.Generator(device=dev).manual_seed(1)
    delta2 = torch.rand(T2, generator=g, device=dev)
    idx2 = torch.empty(T2, dtype=torch.int32, device=dev)
    sel_ws2 = torch.empty(L.dash_select_workspace_size(T2), dtype=torch.uint8, device=dev)
    K2 = math.floor(0.5 * T2)
    cases = {
        "score_abs": (lambda: dash.score(U, out=delta), T * d * 2 + 4 * T),
        "score_rel": (lambda: dash.score(U, H, relative=True, out=delta_r), 2 * T * d * 2 + 4 * T),
        "select_topk_keep0.5": (select_call("topk", 0.5, 0.0), 4 * T + 4 * K + 4),
        "select_threshold_median": (select_call("threshold", 0.0, med), 4 * T + 4 * (T // 2) + 4),
        "gather_K16384": (lambda: dash.compact(U, sel), 2 * K * d * 2 + 4 * K),
        "select_topk_keep0.5_T131072": (
            lambda: L.dash_select(dash._p(delta2), T2, dash.SELECTS["topk"], 0.5, 0.0, 0, 0, dash._p(idx2), None,
                                  dash._p(count), dash._p(sel_ws2), sel_ws2.numel(), None), 4 * T2 + 4 * K2 + 4),
    }
    out = {}
    for name, (fn, nbytes) in cases.items():
        ms = cold(fn)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"us": ms * 1e3, "bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}
    dash.check_device()
    out["workload"] = ("U, H bf16 [32768, 3584] N(0,1), 3264 rows of U x4 in 51 spans of 64 (seed 1); "
                       "top-k keep 0.5 (K = 16384) and threshold = median delta; top-k keep 0.5 also over "
                       "131072 uniform scores")
    out["timing"] = f"each launch alone after a 256 MB L2-flushing write, median of {reps}"
    del U, H, flush
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ ours
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="qwen7b-32k", choices=sorted(WORKLOADS))
    ap.add_argument("--mode", default=None, choices=["prune", "halt"], help="default: the workload's mode")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the dense / other-mode / e2e / fp16 / 128K / score-select legs")
    ap.add_argument("--no-decode", action="store_true", help="skip the generation leg")
    ap.add_argument("--no-128k", action="store_true", help="skip the T=131072 leg")
    args = ap.parse_args()
    if args.impl == "reference":
        # rank 0 alone times the oracle on the host cores; the other ranks exit at once
        world, rank, _ = dist_env()
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    from long_context_prefill_tcgen05_b200 import build, dash
    if rank == 0:
        build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    dims, T = wl["dims"], wl["T"]
    args.mode = args.mode or wl["mode"]
    peaks = load_peaks()

    layers = inputs.make_layers(dims, seed=0, device=dev)
    stack = dash.Stack(dims, layers)
    varlen = wl.get("varlen", False)
    cu = None
    if varlen:
        h0, cu_t = inputs.make_varlen_hidden(n_seq=wl["nseq"], seq_len=T // wl["nseq"], d=dims.d_model, device=dev)
        cu = cu_t.tolist()
    else:
        h0, _ = inputs.make_hidden(T, dims.d_model, seed=0, device=dev, span_rows=wl["span_rows"],
                                   span_len=wl["span_len"])
    pf = Prefill(dash, stack, h0, cu, world)
    threshold = pf.calibrate_threshold(wl, args.mode) if wl.get("calibrate") else 0.0
    cfg = dash.make_config(halt_layer=wl["halt_layer"], mode=args.mode, select=wl["select"], keep=wl["keep"],
                           threshold=threshold, relative=wl["relative"])
    cfg_dense = dash.make_config(mode="dense")

    for _ in range(args.warmup):
        pf.step(cfg)
    dash.check_device()
    # The headline: K steps with no per-launch instrumentation.
    clock = ClockSampler(local)
    clock.start()
    ms, K, _ = pf.timed(cfg, args.steps)
    clocks = clock.stop()
    dash.check_device()
    active = pf.idx[:K].cpu().numpy()
    halted_flops, pairs_by_rows = work_accounting(dims, T, cu, args.mode, wl["halt_layer"], K, active)
    value = world * T / (ms / 1e3)
    # A separate instrumented pass (CUDA events around every launch) gives the
    # per-kernel breakdown and the dominant kernel's roofline.
    n_rec = 2
    _, _, recs = pf.timed(cfg, n_rec, record=True)
    kernels, roof, launches_per_step = kernel_breakdown(recs, dims, pairs_by_rows, n_rec, peaks)
    roof["step_tflops"] = halted_flops / (ms / 1e3) / 1e12

    extra = {}
    if not args.no_extra:
        dense_flops = costs.varlen_prefill_flops(dims, cu) if varlen else costs.prefill_flops(dims, T)
        other = "halt" if args.mode == "prune" else "prune"
        cfg_o = dash.make_config(halt_layer=wl["halt_layer"], mode=other, select=wl["select"], keep=wl["keep"],
                                 threshold=threshold, relative=wl["relative"])
        # Dense, this mode and the other mode are timed in alternating single
        # steps (medians over the rounds), so a drift of the power-capped clock
        # during the run does not bias their ratios.
        pf.step(cfg_dense)
        pf.step(cfg_o)
        legs = [(cfg_dense, []), (cfg, []), (cfg_o, [])]
        for r in range(max(3, args.steps)):
            for c, times in legs[r % 3:] + legs[:r % 3]:
                times.append(pf.timed(c, 1)[0])
        ms_d, ms_m, ms_o = (statistics.median(t) for _, t in legs)
        _, K_o, _ = pf.timed(cfg_o, 1)  # the other mode's active set, for its FLOP count
        flops_o, _ = work_accounting(dims, T, cu, other, wl["halt_layer"], K_o, pf.idx[:K_o].cpu().numpy())
        extra = {
            "dense": {"tokens_per_s": world * T / (ms_d / 1e3), "ms_per_step": ms_d,
                      "tflops": dense_flops / (ms_d / 1e3) / 1e12},
            other + "_mode": {"tokens_per_s": world * T / (ms_o / 1e3), "ms_per_step": ms_o, "K": K_o,
                              "speedup_vs_dense": ms_d / ms_o,
                              "flop_bound": dense_flops / flops_o},
            "speedup_vs_dense": ms_d / ms_m,
            "flop_bound": dense_flops / halted_flops,
            "interleaved": {"rounds": len(legs[0][1]), "ms_per_step": {"dense": ms_d, args.mode: ms_m, other: ms_o},
                            "note": "median of single steps alternating dense / this mode / the other mode"},
        }
        # End to end through the C ABI from pinned host memory, as a serving
        # loop runs it: the residual stream is double-buffered, so step i+1's
        # input goes up and step i's result (the K active rows) comes back on
        # a copy stream while step i computes.  Every step's copies are inside
        # the timed region; only the first upload and the last read-back are
        # not hidden behind a prefill.
        h_host = h0.cpu().pin_memory()
        out_host = torch.empty(T, dims.d_model, dtype=torch.bfloat16).pin_memory()
        comp, copy = torch.cuda.Stream(), torch.cuda.Stream()
        bufs = [pf.H, torch.empty_like(pf.H)]
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]

        def e2e_run(n):
            rows = T
            with torch.cuda.stream(copy):
                bufs[0].copy_(h_host, non_blocking=True)
                ready[0].record(copy)
            for i in range(n):
                cur, nxt = bufs[i % 2], bufs[(i + 1) % 2]
                if i + 1 < n:  # nxt's last read-back is already queued ahead on this stream
                    with torch.cuda.stream(copy):
                        nxt.copy_(h_host, non_blocking=True)
                        ready[(i + 1) % 2].record(copy)
                comp.wait_event(ready[i % 2])
                k = pf.run(cfg, H=cur, stream=comp)
                done[i % 2].record(comp)
                rows = k if args.mode == "prune" else T
                copy.wait_event(done[i % 2])
                with torch.cuda.stream(copy):
                    out_host[:rows].copy_(cur[:rows], non_blocking=True)
            return rows
        e2e_run(2)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(2, args.steps)
        e0.record(copy)
        rows = e2e_run(n_e2e)
        e1.record(copy)
        torch.cuda.synchronize()
        ms_e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        extra["e2e"] = {"value": world * T / (ms_e / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": T * dims.d_model * 2, "d2h_bytes_per_step": rows * dims.d_model * 2}
        del bufs, h_host, out_host
        torch.cuda.empty_cache()

        def pf16_of():
            s16 = dash.Stack(dims, [{k: v.half() for k, v in w.items()} for w in layers])
            return Prefill(dash, s16, h0.half(), cu, world)
        extra["fp16"] = fp16_leg(dash, wl, dims, h0, cu, cfg, pf16_of, pf, world)
        if args.workload == "qwen7b-32k" and not args.no_128k:
            extra["t128k"] = long_context_leg(dash, stack, dims, dev, peaks, world)
        extra["score_select"] = score_select_leg(dash, dev, peaks)
    dash.check_device()
    if not args.no_decode:
        # the cache of a prune-mode prefill with the workload's selection
        cfg_cache = dash.make_config(halt_layer=wl["halt_layer"], mode="prune", select=wl["select"],
                                     keep=wl["keep"], threshold=threshold, relative=wl["relative"])
        extra["decode"] = decode_leg(dash, stack, dims, wl, h0, cu, cfg_cache, cfg_dense, dev, peaks)
        dash.check_device()

    wbytes = dims.n_layers * costs.layer_weight_bytes(dims)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random-init weights, N(0,1) inputs)",
        "config": {"workload": wl["name"], "global_batch": world * wl.get("nseq", 1), "seq_len": T,
                   "halt_layer": wl["halt_layer"], "keep": wl["keep"], "mode": args.mode, "select": wl["select"],
                   **({"threshold": threshold} if wl["select"] == "threshold" else {}),
                   "parallelism": f"replicas x{world}",
                   "l2": (f"inputs larger than L2 ({wbytes / 1e9:.1f} GB of weights per step)" if wbytes > 126e6 else
                          "inputs fit in L2 (a small parity workload, not a headline figure)")},
        "K": K, "halted_tflop_per_step": halted_flops / 1e12,
        "gpu_launches": launches_per_step * args.steps, "roofline": roof, "kernels": kernels,
        "kernels_timing": f"separate pass of {n_rec} steps with CUDA events around every launch",
        "clocks": clocks,
    }
    out.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(dims, T, halted_flops)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
