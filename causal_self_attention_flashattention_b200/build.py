"""Builds libgpt2attn.so (sm_100a) in-tree with nvcc.

    python -m causal_self_attention_flashattention_b200.build [--verbose]

The library is built from the CUDA translation units in csrc/ (gpt2attn.cu,
which includes the kernel headers, and noalloc.cu), linked with the static
CUDA runtime. It does not link against
libcuda: the tensor-map encoder is fetched at run time through
cudaGetDriverEntryPoint. Cross-compiling needs no GPU.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libgpt2attn.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA 12.9 toolkit is required to build the library")


def sources() -> list[str]:
    files = [os.path.join(INCLUDE, "gpt2attn.h")]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            files.append(os.path.join(CSRC, name))
    return files


def is_stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(f) > t for f in sources())


def build(verbose: bool = False, force: bool = False) -> str:
    """Compiles the library if it is missing or older than its sources."""
    if not force and not is_stale():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [
        _nvcc(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo",
        "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
        f"-I{INCLUDE}", f"-I{CSRC}",
        "-o", tmp, *[os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith(".cu")],
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    path = build(verbose="--verbose" in sys.argv, force="--force" in sys.argv)
    print(path)
