"""Build libmla_b200.so in-tree with nvcc for sm_100a (no GPU needed).

build() makes the product library.  build(trace=True) makes
libmla_b200_trace.so from the same sources with MLA_TRACE defined: the decode
kernel then records per-tile timestamps into a buffer given through
mla_debug_set_trace_buffer (see trace.py); everything else is identical.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["api.cu", "decode.cu", "metadata.cu", "combine.cu", "noalloc.cu", "append.cu"]
HEADERS = ["common.cuh", "sm100.cuh", "append.cuh", "entry.cuh"]
OUT = os.path.join(HERE, "libmla_b200.so")
OUT_TRACE = os.path.join(HERE, "libmla_b200_trace.so")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def build(verbose: bool = False, force: bool = False, trace: bool = False) -> str:
    out = OUT_TRACE if trace else OUT
    srcs = [os.path.join(HERE, "csrc", s) for s in SOURCES]
    deps = srcs + [os.path.join(HERE, "csrc", h) for h in HEADERS] + \
        [os.path.join(HERE, "..", "include", "mla.h")]
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-o", out + ".tmp", *srcs]
    if trace:
        cmd.insert(1, "-DMLA_TRACE")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(out)}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True, trace="--trace" in sys.argv))
