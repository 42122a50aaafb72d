"""Builds libhstu.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m hstu_sequential_transducer_layer_b200.build [--force] [--ptxas-info]

Objects go to <repo>/_build/; the shared library is written next to this
file so that it travels with the source tree.  The CUDA runtime is linked
statically and the driver API is reached through the runtime's entry-point
query, so the library loads on a machine without a GPU driver.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libhstu.so")

SOURCES = ["runtime.cu", "api.cu", "sched.cu", "gemm_tc.cu", "attn_tc.cu", "simt_f32.cu",
           "noalloc.cu", "sl.cu", "retrieval.cu", "transformer.cu", "attn_bwd.cu", "bwd.cu"]
HEADERS = [os.path.join(CSRC, "ptx.cuh"), os.path.join(CSRC, "hstu_internal.h"),
           os.path.join(INCLUDE, "hstu.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "--expt-relaxed-constexpr", "-I" + INCLUDE]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libhstu.so")
    return p


def _digest(paths, extra) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(extra).encode())
    return h.hexdigest()[:16]


def _compile(src: str, ptxas_info: bool, force: bool) -> tuple[str, str]:
    path = os.path.join(CSRC, src)
    flags = NVCC_FLAGS + (["-Xptxas", "-v"] if ptxas_info else [])
    tag = _digest([path] + HEADERS, flags)
    obj = os.path.join(BUILD, f"{os.path.splitext(src)[0]}.{tag}.o")
    if os.path.exists(obj) and not force and not ptxas_info:
        return obj, ""
    cmd = [nvcc()] + flags + ["-c", path, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda s: _compile(s, ptxas_info, force), SOURCES))
    objs = [o for o, _ in results]
    if ptxas_info or verbose:
        for (o, log), s in zip(results, SOURCES):
            if log:
                sys.stderr.write(f"== {s}\n{log}")
    link_tag = _digest(objs, ["link"])
    stamp = os.path.join(BUILD, "libhstu.stamp")
    if (not force and os.path.exists(LIB) and os.path.exists(stamp)
            and open(stamp).read() == link_tag):
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-cudart", "static", "-lpthread",
                                                              "-ldl", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(link_tag)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_info=a.ptxas_info, verbose=True))
