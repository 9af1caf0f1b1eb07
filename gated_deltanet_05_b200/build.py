"""Build libgdn_b200.so in-tree with nvcc for sm_100a (B200).

    python -m gated_deltanet_05_b200.build [--verbose-ptxas]

The library is a single translation unit (csrc/gdn_lib.cu) exporting the C ABI of
include/gdn.h. Cross-compiles without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC_DIR = os.path.join(PKG, "csrc")
MAIN = os.path.join(SRC_DIR, "gdn_lib.cu")
OUT = os.path.join(PKG, "libgdn_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _sources():
    out = [os.path.join(ROOT, "include", "gdn.h")]
    for f in sorted(os.listdir(SRC_DIR)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not needs_build():
        return OUT
    cmd = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), "-o", OUT, MAIN]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(OUT)
