"""Build ``libwq.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

A second build, ``libwq_shortwait.so``, compiles the same sources with a
pipeline-wait limit of 0 (``WQ_PIPE_WAIT_NS``) and the test hook
``wq_test_expire_wait`` (``WQ_TEST_HOOKS``): a kernel whose bounded wait is on
a barrier nothing arrives on.  Only the tests load it, to check that an
expired wait is reported as WQ_ERR_DEVICE_TIMEOUT and leaves the GPU usable.

Each ``csrc/*.cu`` translation unit is compiled for ``sm_100a`` only, the CUDA
runtime is linked statically and the CUDA driver API is reached at run time
through ``cudaGetDriverEntryPoint``, so the library loads on a host without a
GPU driver (its symbols can be inspected there) and needs only a B200 to run.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libwq.so")
VARIANTS = {"": [], "shortwait": ["-DWQ_PIPE_WAIT_NS=0ull", "-DWQ_TEST_HOOKS"]}


def lib_path(variant: str = "") -> str:
    return os.path.join(HERE, f"libwq_{variant}.so" if variant else "libwq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(HERE, "..", "include", "wq.h"), __file__]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra=(), variant: str = "") -> str:
    """Build one library (``variant`` "" for libwq.so); returns its path."""
    lib = lib_path(variant)
    if not force and not _stale(lib):
        return lib
    bdir = os.path.join(BUILD, variant) if variant else BUILD
    os.makedirs(bdir, exist_ok=True)
    vflags = VARIANTS[variant]

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *vflags, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose:
        for _, err in results:
            sys.stderr.write(err)
    objs = [o for o, _ in results]
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-Xcompiler", "-fPIC",
           "-Xlinker", "--no-undefined", *objs, "-o", tmp, "-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def build_all(force: bool = False) -> None:
    for v in VARIANTS:
        build(force=force, variant=v)


if __name__ == "__main__":
    for v in VARIANTS:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, variant=v))
