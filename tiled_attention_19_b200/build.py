"""Build the CUDA library in-tree: tiled_attention_19_b200/libattn_b200.so (sm_100a only).

nvcc cross-compiles for sm_100a without a GPU, so this runs on any host with the CUDA
toolkit. The library is one translation unit (csrc/api.cu) plus headers; the CUDA
runtime is linked statically so the .so does not depend on the runtime version that
other libraries in the process bring.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libattn_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libattn_b200.so")


def sources() -> list[str]:
    out = [os.path.join(INCLUDE, "attn.h")]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    return out


def is_stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc_cmd(out: str, extra: list[str] | None = None) -> list[str]:
    return [nvcc_path(), "-std=c++17", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
            "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
            "-Xptxas", "-v", "-o", out, os.path.join(CSRC, "api.cu")] + (extra or [])


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not is_stale():
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    proc = subprocess.run(nvcc_cmd(tmp), capture_output=True, text=True)
    log = proc.stdout + proc.stderr
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{log}")
    with open(os.path.join(HERE, "build_ptxas.log"), "w") as f:
        f.write(log)
    if verbose:
        print(log)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
