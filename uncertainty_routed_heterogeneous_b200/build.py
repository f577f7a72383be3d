"""Builds libheta.so (every CUDA source under csrc/) for sm_100a, in-tree.

    python -m uncertainty_routed_heterogeneous_b200.build [--force] [--verbose-ptxas]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (in parallel),
then linked into ``uncertainty_routed_heterogeneous_b200/libheta.so``.  nvcc
cross-compiles without a GPU.  The CUDA runtime is linked statically and the
driver entry point for tensor-map encoding is fetched at run time, so the
library needs no libcuda at link time.  The plain-C example
``examples/heta_run.c`` (the path driven through ``include/heta.h`` alone) is
built next to it as ``examples/heta_run``.
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libheta.so")
EXAMPLE_SRC = os.path.join(PKG, "examples", "heta_run.c")
EXAMPLE = os.path.join(PKG, "examples", "heta_run")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, ptxas_verbose):
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC] + ARCH + FLAGS + ["-c", src, "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed on %s:\n%s\n%s" % (src, r.stdout, r.stderr))
    return obj, r.stderr


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True) -> str:
    """Compiles what changed and relinks libheta.so; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    hdrs = _headers()
    todo = [s for s in srcs
            if force or ptxas_verbose or _stale(os.path.join(BUILD, os.path.basename(s)[:-3] + ".o"),
                                                [s] + hdrs)]
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(todo)))) as ex:
        for obj, log in ex.map(lambda s: _compile(s, ptxas_verbose), todo):
            if log and (ptxas_verbose or not quiet):
                sys.stderr.write(log)
    objs = [os.path.join(BUILD, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if force or todo or _stale(LIB, objs):
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = [NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, LIB)
    build_example(force)
    return LIB


def build_example(force: bool = False) -> str:
    """gcc-compiles examples/heta_run.c against include/heta.h, libheta.so and
    the CUDA runtime (for its allocations and copies); returns its path."""
    if force or _stale(EXAMPLE, [EXAMPLE_SRC, LIB] + glob.glob(os.path.join(INCLUDE, "*.h"))):
        tmp = EXAMPLE + ".tmp.%d" % os.getpid()
        cmd = [os.environ.get("CC", "gcc"), "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror",
               "-I", INCLUDE, "-I", os.path.join(CUDA_HOME, "include"), EXAMPLE_SRC, "-o", tmp,
               "-L", PKG, "-lheta", "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart", "-lm",
               "-Wl,-rpath,$ORIGIN/..", "-Wl,-rpath," + os.path.join(CUDA_HOME, "lib64")]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("the C example failed to build:\n%s\n%s" % (r.stdout, r.stderr))
        os.replace(tmp, EXAMPLE)
    return EXAMPLE


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv,
                quiet=False))
