"""Builds the in-tree C-ABI shared library ``libmoe_b200.so`` for sm_100a.

Run as ``python -m routing_dispatch_expert_softmax_b200.build``.  nvcc
cross-compiles without a GPU; the library lands next to this file so it
travels with the source tree.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libmoe_b200.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["moe_abi.cu", "moe_routing.cu", "moe_gemm_sm100.cu", "moe_noalloc.cu", "moe_w8a8.cu",
           "moe_eplb.cu", "moe_dedup.cu", "moe_gemm_fp8.cu", "moe_ep.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA 12.9 toolkit is required")
    return cand


def _run(cmd):
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError("command failed:\n" + " ".join(cmd) + "\n" + p.stdout + p.stderr)
    return p.stdout + p.stderr


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    """Compile every .cu for sm_100a and link the shared library."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    nvcc = _nvcc()
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    deps.append(os.path.join(ROOT, "include", "moe.h"))
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) > max(os.path.getmtime(d) for d in deps)):
        return OUT
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    objs = [os.path.join(BUILD_DIR, os.path.basename(s) + ".o") for s in srcs]

    def one(pair):
        src, obj = pair
        return _run([nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj])

    with cf.ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        logs = list(ex.map(one, zip(srcs, objs)))
    tmp = OUT + ".tmp"
    _run([nvcc, *ARCH, "-shared", "-o", tmp, *objs])
    os.replace(tmp, OUT)
    if verbose_ptxas:
        sys.stdout.write("".join(logs))
    return OUT


if __name__ == "__main__":
    path = build(verbose_ptxas="-v" in sys.argv, force="--force" in sys.argv)
    print(path)
