"""Builds liblsh_attention_hash.so in-tree with nvcc for sm_100a.

Usage: python -m lsh_attention_hash_b200.build  (or build() from Python).
The library has one translation unit (csrc/lsh_api.cu includes every kernel
header), links the CUDA runtime statically and exports only the C ABI of
include/lsh_attention_hash.h.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_NAME = "liblsh_attention_hash.so"


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    csrc = os.path.join(PKG, "csrc")
    return [os.path.join(csrc, f) for f in sorted(os.listdir(csrc)) if f.endswith((".cu", ".cuh"))]


def build(verbose: bool = False, force: bool = False) -> str:
    out = os.path.join(PKG, LIB_NAME)
    deps = sources() + [os.path.join(ROOT, "include", "lsh_attention_hash.h")]
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(d) <= t for d in deps):
            return out
    cmd = [
        nvcc_path(), "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-O3", "-lineinfo",
        "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"),
        "-Xptxas", "-warn-spills" if not verbose else "-v",
        "-o", out + ".tmp", os.path.join(PKG, "csrc", "lsh_api.cu"),
    ]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force=True))
