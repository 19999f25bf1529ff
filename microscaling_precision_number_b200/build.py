"""Build libmx.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m microscaling_precision_number_b200.build [--force] [--verbose] [--checked]

Each .cu file under csrc/ is compiled to an object (in parallel) and linked into
``microscaling_precision_number_b200/libmx.so``.  The CUDA runtime is linked statically;
the driver API (tensor-map encoding) is reached through cudaGetDriverEntryPoint, so the
library loads on a machine without a GPU driver (it only fails when a call needs a GPU).

``--checked`` builds ``libmx_checked.so`` instead: the same sources compiled with
-DMX_CHECKED, in which every global store of every kernel is bounds-checked against the
output extents the launchers register (csrc/checked.cuh).  It is a test build, loaded
through the MX_LIB_PATH environment variable.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmx.so")
LIB_CHECKED = os.path.join(PKG, "libmx_checked.so")
SOURCES = ["api.cu", "stream.cu", "quant.cu", "dual.cu", "gemm.cu", "gemm2.cu", "nested.cu", "train.cu", "noalloc.cu"]
HEADERS = ["checked.cuh", "codec.cuh", "nvfp4.cuh", "ptx.cuh", "tiling.cuh", "umma.cuh", "internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    build_dir = os.path.join(BUILD, "checked") if checked else BUILD
    lib_path = LIB_CHECKED if checked else LIB
    os.makedirs(build_dir, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "mx.h")]
    objs = []
    jobs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            cmd = [nvcc()] + ARCH + FLAGS + (["-DMX_CHECKED"] if checked else []) + \
                (["-Xptxas", "-v"] if verbose else []) + ["-c", s, "-o", o]
            jobs.append(cmd)
    with cf.ThreadPoolExecutor(max_workers=min(4, max(1, len(jobs)))) as ex:
        for cmd, res in zip(jobs, ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs)):
            if verbose or res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
            if res.returncode != 0:
                raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if force or jobs or _stale(lib_path, objs):
        tmp = lib_path + f".tmp{os.getpid()}"
        cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-Xlinker", "-z,defs", "-o", tmp] + objs + \
            ["-cudart", "static"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("link failed")
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
