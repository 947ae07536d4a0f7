"""Build the in-tree CUDA library ``libmla_b200.so`` for sm_100a with nvcc.

Usage: ``python -m mla_paged_kv_get_b200.build [--verbose]``.  The shared
object is written next to this file so that it travels with the source tree.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = ["capi.cu", "metadata.cu", "decode.cu", "decode_pair.cu", "combine.cu", "noalloc.cu"]
LIB = os.path.join(HERE, "libmla_b200.so")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, force: bool = False) -> str:
    csrc = os.path.join(HERE, "csrc")
    srcs = [os.path.join(csrc, s) for s in SOURCES]
    deps = srcs + [os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(ROOT, "include", "mla_b200.h"))
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in deps)
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [nvcc_path(), "-shared", "-Xcompiler", "-fPIC", "-O3", "-lineinfo", "-std=c++17",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp"] + srcs
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True))
