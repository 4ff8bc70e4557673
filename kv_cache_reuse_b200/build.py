"""Build libmac_b200.so in-tree with nvcc for sm_100a (B200).

Usage: python -m kv_cache_reuse_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmac_b200.so")
SOURCES = ["mac_api.cu", "mac_match.cu", "mac_attend.cu", "mac_attend_tc.cu", "mac_noalloc.cu"]
HEADERS = [os.path.join(CSRC, "mac_internal.cuh"), os.path.join(CSRC, "mac_match_dev.cuh"),
           os.path.join(CSRC, "mac_attend_dev.cuh"),
           os.path.join(ROOT, "include", "mac.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu for sm_100a (the files in parallel) and link the shared
    library; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    objs, cmds = [], []
    nvcc = _nvcc()
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + HEADERS):
            cmds.append([nvcc] + ARCH + FLAGS + ["-c", s, "-o", o])
    for cmd in cmds:
        if verbose:
            print(" ".join(cmd))
    with ThreadPoolExecutor(max_workers=max(1, len(cmds))) as ex:
        for f in [ex.submit(subprocess.check_call, cmd) for cmd in cmds]:
            f.result()
    if force or _stale(LIB, objs):
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [nvcc] + ARCH + ["-shared", "-o", tmp] + objs
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
