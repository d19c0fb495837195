"""Compile the CUDA library (libpa.so) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpa.so")
SOURCES = ["api.cu", "api_static.cu", "plan.cu", "scatter.cu", "smallseq.cu", "smallseq_bwd.cu",
           "decode.cu", "decode_sliced.cu", "prefill_sm100.cu"]
HEADERS = ["common.cuh", "decode.cuh", "kernels.h", "layout.h", "spans.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "pa.h"))
    deps.append(__file__)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Build libpa.so if any source is newer than it; returns its path.

    Each source compiles to an object in its own nvcc process (in parallel),
    then one nvcc call links the shared library."""
    if not force and not _stale():
        return LIB
    import concurrent.futures
    import tempfile
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
             "-Xcompiler", "-fPIC"]
    if ptxas_info:
        flags += ["-Xptxas", "-v"]
    with tempfile.TemporaryDirectory(prefix="pa_build_") as tmpdir:
        objs = [os.path.join(tmpdir, os.path.splitext(src)[0] + ".o") for src in SOURCES]

        def compile_one(i):
            cmd = [_nvcc(), *flags, "-c", os.path.join(CSRC, SOURCES[i]), "-o", objs[i]]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            subprocess.check_call(cmd, cwd=CSRC)

        workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
            list(pool.map(compile_one, range(len(SOURCES))))
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = [_nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd, cwd=CSRC)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv)
    print(LIB)
