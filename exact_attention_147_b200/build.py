"""Build libfa2.so (the CUDA kernels and the C ABI) in-tree with nvcc.

Usage:  python -m exact_attention_147_b200.build [--verbose]

The library is compiled for sm_100a only; cudart is linked statically, so the
.so loads on a machine without a GPU (calls then return FA2_ERR_CUDA after
their argument checks).
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "fa2_api.cu")
OUT = os.path.join(HERE, "libfa2.so")
HEADERS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))
           if f.endswith((".cuh", ".cu", ".h"))] + [os.path.join(ROOT, "include", "fa2.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(h) > t for h in HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libfa2.so if it is missing or older than its sources."""
    if not force and not needs_build():
        return OUT
    tmp = OUT + ".tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, "-o", tmp, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(OUT)
