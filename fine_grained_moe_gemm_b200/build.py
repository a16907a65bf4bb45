"""Builds the in-tree CUDA libraries (sm_100a) with nvcc: ``libmoe_b200.so`` and
``libmoe_b200_debug.so``, the same sources compiled with MOE_DEBUG (the
checking build: table-dependent accesses are checked against their buffers
and flagged with MOE_DEVERR_BOUNDS)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe_b200.so")
LIB_DEBUG = os.path.join(HERE, "libmoe_b200_debug.so")
SOURCES = ["moe_kernels.cu", "moe_api.cu", "moe_noalloc.cu"]
HEADERS = ["moe_device.cuh", "moe_gemm.cuh", "moe_gemm_fp8.cuh", "moe_gemm2.cuh", "moe_gemm2_fp8.cuh", "moe_launch.h", os.path.join("..", "..", "include", "moe.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def _build_variants(variants, verbose: bool, ptxas_verbose: bool) -> None:
    """Compiles every (variant, source) object in parallel, then links each library."""
    jobs, variants_objs = [], []
    for lib, defines, sub in variants:
        build_dir = os.path.join(HERE, "_build", sub)
        os.makedirs(build_dir, exist_ok=True)
        objs = []
        for src in SOURCES:
            obj = os.path.join(build_dir, src.replace(".cu", ".o"))
            cmd = [_nvcc(), *NVCC_FLAGS, *defines, "-c", os.path.join(CSRC, src), "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            jobs.append((subprocess.Popen(cmd), cmd))
            objs.append(obj)
        variants_objs.append((lib, objs))
    failed = [cmd for proc, cmd in jobs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    for lib, objs in variants_objs:
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([_nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp,
                        "-lcudart", "-ldl"], check=True)
        os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    """Builds whichever of the two libraries is missing or older than its sources
    (both with force); returns the path of the regular one."""
    todo = [(LIB, [], "release"), (LIB_DEBUG, ["-DMOE_DEBUG"], "debug")]
    todo = [v for v in todo if force or _stale(v[0])]
    if todo:
        _build_variants(todo, verbose, ptxas_verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_verbose="-v" in sys.argv))
