"""Builds libfluxbin.so (sm_100a) in-tree with nvcc / g++.

Objects go to ``_build/`` at the repository root; the shared library lands
next to this file so that it travels with the source tree.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfluxbin.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")] + ARCH
CXX_FLAGS = ["-O3", "-std=c++17", "-fPIC", "-Wall", "-pthread", "-I", os.path.join(ROOT, "include")]

CU_SOURCES = ["fluxbin_api.cu", "fluxbin_inst_mu8.cu", "fluxbin_inst_mu4.cu", "fluxbin_inst_tc.cu",
              "fluxbin_inst_lut1.cu", "fluxbin_inst_lut1h.cu"]
CXX_SOURCES = ["fluxbin_pack.cpp", "fluxbin_fit.cpp"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _sources():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC)]


def _source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for p in sorted(_sources()) + [os.path.join(ROOT, "include", "fluxbin.h"), os.path.abspath(__file__)]:
        h.update(os.path.basename(p).encode())
        h.update(open(p, "rb").read())
    return h.hexdigest()


def _stale() -> bool:
    """Rebuild when the library is missing or was built from other sources
    (content hash, so copying the tree elsewhere does not force a rebuild)."""
    if not os.path.exists(LIB) or not os.path.exists(LIB + ".srchash"):
        return True
    return open(LIB + ".srchash").read().strip() != _source_hash()


def _compile(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("build failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    return r.stderr


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not ptxas_info and not _stale():
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    nvcc = _nvcc()
    jobs, objs = [], []
    for f in CU_SOURCES:
        o = os.path.join(OUT_DIR, f + ".o")
        extra = ["-Xptxas", "-v"] if ptxas_info else []
        jobs.append([nvcc, *NVCC_FLAGS, *extra, "-c", os.path.join(CSRC, f), "-o", o])
        objs.append(o)
    for f in CXX_SOURCES:
        o = os.path.join(OUT_DIR, f + ".o")
        jobs.append(["g++", *CXX_FLAGS, "-c", os.path.join(CSRC, f), "-o", o])
        objs.append(o)
    with cf.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        logs = list(ex.map(_compile, jobs))
    tmp = LIB + f".tmp{os.getpid()}"
    _compile([nvcc, "-shared", *ARCH, "-o", tmp, *objs, "-lcudart_static", "-lrt", "-lpthread", "-ldl"])
    os.replace(tmp, LIB)
    with open(LIB + ".srchash", "w") as f:
        f.write(_source_hash() + "\n")
    if verbose or ptxas_info:
        for lg in logs:
            if lg.strip():
                sys.stderr.write(lg)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
    print(LIB)
