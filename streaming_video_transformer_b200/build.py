"""Builds libsvt.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m streaming_video_transformer_b200.build [--verbose]

No GPU is needed: nvcc cross-compiles.  The library lands next to this file
so that it travels with the source tree.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsvt.so")
SOURCES = ["svt_cache.cu", "svt_kernels.cu", "svt_attn_sm100.cu", "svt_noalloc.cu",
           "svt_selftest.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# The D = 64 attention kernel splits its registers between two warpgroups
# (setmaxnreg 64 / 192) out of the 256 x 128 it is launched with; the split
# only adds up when ptxas gives the kernel exactly this many registers, and
# otherwise the increase would wait for registers that never come.
SPLIT_KERNEL = "attn_sm100_kernelILi64E"
SPLIT_LAUNCH_REGS = 128


def check_register_split(ptxas_log: str) -> None:
    """Raise unless every D = 64 attention kernel was compiled with exactly
    SPLIT_LAUNCH_REGS registers (see the warpgroup split in the kernel)."""
    counts = []
    current = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current and SPLIT_KERNEL in current:
            counts.append(int(m.group(1)))
            current = None
    if not counts:
        raise RuntimeError("ptxas report has no D = 64 attention kernel")
    bad = [c for c in counts if c != SPLIT_LAUNCH_REGS]
    if bad:
        raise RuntimeError(f"D = 64 attention kernel compiled with {bad} registers, not "
                           f"{SPLIT_LAUNCH_REGS}: its warpgroup register split would not add up")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, force: bool = False) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(ROOT, "include", "svt.h"))
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in deps)):
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-Xptxas=-v", "-I", os.path.join(ROOT, "include"),
           "--expt-relaxed-constexpr", "-o", LIB + ".tmp", *srcs]
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed")
    if verbose:
        sys.stderr.write(r.stderr)
    try:
        check_register_split(r.stdout + r.stderr)
    except RuntimeError:
        os.remove(LIB + ".tmp")
        raise
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
