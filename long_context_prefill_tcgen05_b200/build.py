"""Builds libdash.so (the sm_100a CUDA library) in-tree with nvcc.

    python -m long_context_prefill_tcgen05_b200.build [--force] [--verbose]
"""
import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdash.so")
MAIN = os.path.join(CSRC, "dash_api.cu")

NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-I" + INCLUDE,
]


def _sources():
    return (glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def source_hash():
    h = hashlib.sha256()
    h.update(" ".join(FLAGS[:-1]).encode())
    for s in sorted(_sources()):
        h.update(os.path.basename(s).encode())
        with open(s, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def up_to_date():
    """True when libdash.so exists and was built from the current sources."""
    stamp = LIB + ".srchash"
    if not (os.path.exists(LIB) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == source_hash()


def build(force=False, verbose=False, ptxas_info=False):
    """Compile libdash.so unless it is newer than every source.  Raises on failure."""
    if not force and up_to_date():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if ptxas_info else []) + ["-o", tmp, MAIN]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stderr[-8000:]}")
    if verbose or ptxas_info:
        sys.stderr.write(r.stderr)
    os.replace(tmp, LIB)
    with open(LIB + ".srchash", "w") as f:
        f.write(source_hash())
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
