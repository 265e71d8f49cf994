"""Builds ``libattn.so`` in-tree with nvcc for sm_100a (B200).

Usage: ``python -m online_softmax_attention_fwd_b200.build [--force] [--ptxas-verbose]``.
Objects go to ``_build/`` at the repository root; the shared library is written next to this file,
where the Python binding loads it from.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(HERE, "libattn.so")
FAULT_LIB_PATH = os.path.join(HERE, "libattn_faultinject.so")  # test-only build, see build()
SOURCES = ["api.cu", "simt.cu", "decode.cu", "decode_static.cu", "fwd_sm100.cu", "bwd_sm100.cu", "merge.cu"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH_FLAGS + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE,
                       "-Xcompiler", "-Wall", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or "/usr/local/cuda/bin/nvcc"
    return cand if os.path.exists(cand) else "nvcc"


def _deps():
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return hdrs + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def _stale(target: str, inputs) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(x) > t for x in inputs)


def _compile(src: str, force: bool, ptxas_verbose: bool, fault_inject: bool = False) -> str:
    sub = os.path.join(BUILD_DIR, "faultinject") if fault_inject else BUILD_DIR
    obj = os.path.join(sub, os.path.splitext(src)[0] + ".o")
    srcp = os.path.join(CSRC, src)
    if force or _stale(obj, [srcp] + _deps()):
        flags = CFLAGS + (["-DATTN_FAULT_INJECT"] if fault_inject else [])
        cmd = [nvcc()] + flags + (["-Xptxas", "-v"] if ptxas_verbose else []) + ["-c", srcp, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if ptxas_verbose:
            sys.stderr.write(r.stderr)
    return obj


def _link(objs, target: str, force: bool) -> None:
    if force or _stale(target, objs):
        cmd = [nvcc()] + ARCH_FLAGS + ["-shared", "-o", target] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link libattn.so, and the test-only
    fault-injection build libattn_faultinject.so (the same sources with ATTN_FAULT_INJECT: short
    wait limits and a switch that makes one producer skip one copy, for the timeout tests). Returns
    the path of libattn.so."""
    os.makedirs(os.path.join(BUILD_DIR, "faultinject"), exist_ok=True)
    jobs = [(s, False) for s in SOURCES] + [(s, True) for s in SOURCES]
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        objs = list(ex.map(lambda j: _compile(j[0], force, ptxas_verbose and not j[1], j[1]), jobs))
    _link(objs[:len(SOURCES)], LIB_PATH, force)
    _link(objs[len(SOURCES):], FAULT_LIB_PATH, force)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, ptxas_verbose=args.ptxas_verbose))
