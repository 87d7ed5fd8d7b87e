"""Build libmoe_b200.so (sm_100a) in-tree with nvcc.

    python -m mxfp4_latent_moe_router_b200.build [--force]

Objects go to ``_build/`` at the repository root; the shared library lands
next to this file so it travels with the source tree.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libmoe_b200.so")
SOURCES = ["moe_kernels.cu", "moe_k_front.cu", "moe_k_egu.cu", "moe_k_edn.cu",
           "moe_k_tail.cu", "moe_k_mega.cu", "moe_pack.cu", "moe_api.cu", "moe_static.cu"]
HEADERS = ["ptx.cuh", "layout.cuh", "engine.cuh", "topk.cuh", "umma.cuh", "moe_engine.cuh", "moe_mega.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _mtime(p: str) -> float:
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _deps_mtime() -> float:
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "moe.h")]
    return max(_mtime(h) for h in hdrs)


def _compile(src: str, force: bool) -> str:
    s = os.path.join(CSRC, src)
    o = os.path.join(OBJ, src.replace(".cu", ".o"))
    if force or _mtime(o) < max(_mtime(s), _deps_mtime()):
        cmd = [NVCC, *FLAGS, "-c", s, "-o", o + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(o + ".tmp", o)
    return o


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, force), SOURCES))
    if force or _mtime(LIB) < max(_mtime(o) for o in objs):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
               *objs, "-o", tmp]
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    if verbose:
        print(LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
