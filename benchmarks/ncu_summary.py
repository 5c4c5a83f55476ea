"""Summarises an ncu launch list (``--metrics gpu__time_duration.sum --csv``)
of a bench.py run: per kernel, the launches, total time and share of the last
complete prefill step -- the launches between the last two RoPE-table builds
(every prefill starts with one), since a capture limit (-c) may cut the final
step short; with a single build, the launches from it to the end.

    python benchmarks/ncu_summary.py launches.csv
"""
import collections
import csv
import sys

SHORT = [
    ("decode_attn_kernel", "decode_attention"), ("decode_merge_kernel", "decode_merge"),
    ("gemv_kernel<0", "gemv_qkv_rope_append"), ("gemv_kernel<1", "gemv_resid (o_proj / down)"),
    ("gemv_kernel<2", "gemv_gate_up_swiglu"), ("kv_store_kernel", "kv_store"),
    ("attn_kernel", "attention"),
    ("gemm_kernel<256, 4,", "gemm_qkv_rope"), ("gemm_kernel<128, 4,", "gemm_qkv_rope"),
    ("gemm_kernel<256, 2,", "gemm_o_resid_delta"), ("gemm_kernel<128, 2,", "gemm_o_resid_delta"),
    ("gemm_kernel<256, 3,", "gemm_gate_up_swiglu"), ("gemm_kernel<128, 3,", "gemm_gate_up_swiglu"),
    ("gemm_kernel<256, 1,", "gemm_resid (o_proj / down)"), ("gemm_kernel<128, 1,", "gemm_resid (o_proj / down)"),
    ("gemm_kernel<256, 0,", "gemm_store"), ("gemm_kernel<128, 0,", "gemm_store"),
    ("gemm_pair_kernel<4,", "gemm_qkv_rope"), ("gemm_pair_kernel<2,", "gemm_o_resid_delta"),
    ("gemm_pair_kernel<3,", "gemm_gate_up_swiglu"), ("gemm_pair_kernel<1,", "gemm_resid (o_proj / down)"),
    ("gemm_pair_kernel<0,", "gemm_store"),
    ("rmsnorm_kernel", "rmsnorm"), ("score_from_ssq", "score"), ("score_kernel", "score"),
    ("select_kernel", "select"), ("sel_hist_kernel", "select"), ("sel_scan_kernel", "select"),
    ("sel_resolve_kernel", "select"), ("sel_compact_kernel", "select"), ("move_rows_kernel<false>", "gather"), ("move_rows_kernel<true>", "scatter"),
    ("move_rows_kernel<0>", "gather"), ("move_rows_kernel<1>", "scatter"),
    ("rope_table_kernel", "rope_table"),
]


def short(name):
    for key, s in SHORT:
        if key in name:
            return s
    return "other: " + name.split("(")[0][:60]


def load(path):
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr = rows[hi]
    ki, mi, vi = hdr.index("Kernel Name"), hdr.index("Metric Name"), hdr.index("Metric Value")
    ui = hdr.index("Metric Unit")
    scale = {"ns": 1e-6, "us": 1e-3, "usecond": 1e-3, "ms": 1.0, "msecond": 1.0, "nsecond": 1e-6}
    out = []
    for r in rows[hi + 1:]:
        if len(r) > vi and r[mi] == "gpu__time_duration.sum":
            out.append((r[ki], float(r[vi].replace(",", "")) * scale.get(r[ui], 1e-6)))
    return out


def summarise(path):
    launches = load(path)
    starts = [i for i, (n, _) in enumerate(launches) if "rope_table_kernel" in n]
    if len(starts) >= 2:
        step = launches[starts[-2]:starts[-1]]
    else:
        step = launches[starts[-1]:] if starts else launches
    agg = collections.OrderedDict()
    for name, ms in step:
        k = short(name)
        a = agg.setdefault(k, [0, 0.0])
        a[0] += 1
        a[1] += ms
    total = sum(v[1] for v in agg.values())
    lines = [f"{'kernel':34s} {'launches':>8s} {'total ms':>10s} {'share':>7s}"]
    for k, (n, ms) in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        lines.append(f"{k:34s} {n:8d} {ms:10.3f} {ms / total:7.1%}")
    lines.append(f"{'total (one step)':34s} {sum(v[0] for v in agg.values()):8d} {total:10.3f}")
    return "\n".join(lines)


if __name__ == "__main__":
    print(summarise(sys.argv[1]))
