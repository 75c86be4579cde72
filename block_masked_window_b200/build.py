"""Build the sm_100a shared library ``libla_pbd.so`` in-tree with nvcc.

    python -m block_masked_window_b200.build

Every kernel is compiled for ``sm_100a`` only (``-gencode arch=compute_100a,code=sm_100a``)
with ``-lineinfo`` so that profiles map back to source. The CUDA runtime is linked
statically; the CUDA driver is reached at run time through the runtime's entry-point query,
so the library needs no libcuda at link time and builds on a machine without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libla_pbd.so")
SOURCES = ["la_pbd_api.cu", "kv_append.cu", "attn_simt.cu", "attn_tc.cu", "combine.cu",
           "la_pbd_static.cu", "prefill_tc.cu", "noop.cu"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, extra=None):
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v",
           "-I", os.path.join(ROOT, "include"), "-o", out]
    cmd += list(extra or [])
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    return cmd


def build(verbose: bool = False) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    deps.append(os.path.join(ROOT, "include", "la_pbd.h"))
    deps.append(os.path.abspath(__file__))
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in deps):
        return LIB
    tmp = LIB + ".tmp"
    res = subprocess.run(command(tmp), capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose=True))
