"""Build liblighthouse.so in-tree with nvcc for sm_100a (B200).

Each csrc/*.cu is compiled to an object under _build/ (in parallel, skipped
when up to date) and linked into long_context_lh_b200/liblighthouse.so with
the CUDA runtime linked statically, so the library loads on a host without a
GPU driver (only the entry points that launch work need one).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "liblighthouse.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-diag-suppress", "128", "-I", INCLUDE]


def _deps(src: str):
    return [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "lighthouse.h")]


def _compile(src: str, verbose: bool, build_dir: str = BUILD, extra=()) -> str:
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    if os.path.exists(obj) and all(os.path.getmtime(obj) >= os.path.getmtime(d) for d in _deps(src)):
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    os.replace(obj + ".tmp", obj)
    return obj


BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "liblighthouse_debug.so")


def _build_lib(lib: str, build_dir: str, extra, verbose: bool, force: bool) -> str:
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if force:
        for f in glob.glob(os.path.join(build_dir, "*.o")):
            os.remove(f)
    with ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, build_dir, extra), srcs))
    if os.path.exists(lib) and all(os.path.getmtime(lib) >= os.path.getmtime(o) for o in objs):
        return lib
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", lib + ".tmp", *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(lib + ".tmp", lib)
    return lib


def build(verbose: bool = False, force: bool = False) -> str:
    """liblighthouse.so, the library."""
    return _build_lib(LIB, BUILD, (), verbose, force)


def build_debug(verbose: bool = False, force: bool = False) -> str:
    """liblighthouse_debug.so: the same sources with -DLH_DEBUG=1 (bounds checks
    in the kernels, reported through lh_read_device_status)."""
    return _build_lib(LIB_DEBUG, BUILD_DEBUG, ("-DLH_DEBUG=1",), verbose, force)


SELFTEST_SRC = os.path.join(PKG, "selftest", "lh_selftest.cu")
SELFTEST_LIB = os.path.join(PKG, "liblh_selftest.so")


def build_selftest(verbose: bool = False) -> str:
    """liblh_selftest.so: device-helper test hooks, loaded by the tests only."""
    deps = [SELFTEST_SRC] + glob.glob(os.path.join(CSRC, "*.cuh"))
    if os.path.exists(SELFTEST_LIB) and all(os.path.getmtime(SELFTEST_LIB) >= os.path.getmtime(d)
                                            for d in deps):
        return SELFTEST_LIB
    cmd = [NVCC, *ARCH, *FLAGS, "-shared", "-cudart", "static", SELFTEST_SRC, "-o",
           SELFTEST_LIB + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {SELFTEST_SRC}:\n{r.stdout}\n{r.stderr}")
    os.replace(SELFTEST_LIB + ".tmp", SELFTEST_LIB)
    return SELFTEST_LIB


if __name__ == "__main__":
    print(build(verbose=True, force="--force" in sys.argv))
    print(build_debug(verbose=True, force="--force" in sys.argv))
    print(build_selftest(verbose=True))
