"""Build libart.so in-tree (nvcc, sm_100a, CUDA runtime linked statically).

The library is written for the B200 only: one architecture, no PTX fallback.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libart.so")
# one translation unit per group of walk instantiations, so that they compile in parallel
SOURCES = [os.path.join(CSRC, f) for f in ("art_api.cu", "art_order.cu", "art_walk_f32.cu", "art_walk_bf16.cu",
                                           "art_walk_mma.cu", "art_walk_multi.cu", "art_no_alloc.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("art_kernels.cuh", "art_ptx.cuh", "art_host.h", "art_walk.h", "art_walk_dl.cuh", "art_walk_gr.cuh")] + [
    os.path.join(ROOT, "include", "art.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC",
    "-Xptxas", "-warn-spills",
]
LINK_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build_library(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/ into libart.so next to this file if it is missing or
    stale: every translation unit to an object in parallel, then one link."""
    if not force and not stale():
        return LIB
    import tempfile
    from concurrent.futures import ThreadPoolExecutor
    tmpdir = tempfile.mkdtemp(prefix="art_build_")
    objs = [os.path.join(tmpdir, os.path.basename(src)[:-3] + ".o") for src in SOURCES]

    def compile_one(pair):
        src, obj = pair
        cmd = [nvcc(), *NVCC_FLAGS, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        r = subprocess.run(cmd, cwd=CSRC, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
        return cmd, r

    jobs = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with ThreadPoolExecutor(jobs) as ex:
        results = list(ex.map(compile_one, zip(SOURCES, objs)))
    for cmd, r in results:
        if r.stdout:
            sys.stderr.write(r.stdout)
        if r.returncode != 0:
            raise subprocess.CalledProcessError(r.returncode, cmd, r.stdout)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *LINK_FLAGS, "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd, cwd=CSRC)
    os.replace(tmp, LIB)
    for obj in objs:
        os.remove(obj)
    os.rmdir(tmpdir)
    return LIB


if __name__ == "__main__":
    print(build_library(force="--force" in sys.argv, verbose=True))
