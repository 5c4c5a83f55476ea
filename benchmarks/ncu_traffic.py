"""Summarises single-kernel ncu captures taken with
``--metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum --csv``:
per capture, the kernel, its duration and its DRAM bytes read and written,
next to the algorithmic bytes the caller states for that launch.

    python benchmarks/ncu_traffic.py capture.csv ALGORITHMIC_BYTES [capture.csv BYTES ...]
"""
import csv
import sys

UNITS = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9,
         "nsecond": 1e-9, "usecond": 1e-6, "msecond": 1e-3, "ns": 1e-9, "us": 1e-6, "ms": 1e-3, "second": 1.0}


def load(path):
    """{metric: value in bytes or seconds} and the kernel name of the first captured launch."""
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Metric Name" in r)
    hdr = rows[hi]
    ki, mi, ui, vi = (hdr.index(k) for k in ("Kernel Name", "Metric Name", "Metric Unit", "Metric Value"))
    out, name = {}, None
    for r in rows[hi + 1:]:
        if len(r) <= vi:
            continue
        name = name or r[ki]
        if r[ki] != name:
            break
        out[r[mi]] = float(r[vi].replace(",", "")) * UNITS.get(r[ui], 1.0)
    return name, out


def row(path, algo_bytes):
    name, m = load(path)
    t = m["gpu__time_duration.sum"]
    rd, wr = m["dram__bytes_read.sum"], m["dram__bytes_write.sum"]
    return (f"| `{name.split('(')[0][:60]}` | {t * 1e6:.1f} | {rd / 1e6:.1f} | {wr / 1e6:.1f} | "
            f"{algo_bytes / 1e6:.1f} | {(rd + wr) / algo_bytes:.2f} | {algo_bytes / t / 1e9:.0f} |")


if __name__ == "__main__":
    print("| kernel | µs (ncu) | DRAM read MB | DRAM write MB | algorithmic MB | traffic / algorithmic | algorithmic GB/s |")
    print("|---|---|---|---|---|---|---|")
    args = sys.argv[1:]
    for p, b in zip(args[::2], args[1::2]):
        print(row(p, float(b)))
