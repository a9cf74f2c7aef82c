"""Build libcoat.so in-tree with nvcc for sm_100a (B200) only, and its checked
variant libcoat_debug.so (compiled with COAT_DEBUG: every kernel checks the
indices it derives before each access, counts failures on the device and
skips the access; see coat_check_device_error in include/coat.h).

    python -m fp8_optimizer_state_b200.build [--force] [--verbose-ptxas] [--checked]

The library links the CUDA runtime statically, so loading it needs no CUDA
driver (a GPU-less host can load it and check its exports); the first CUDA
call needs one.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libcoat.so")
LIB_CHECKED = os.path.join(HERE, "libcoat_debug.so")
SOURCES = ["api.cu", "adamw_fp8.cu", "codec.cu", "fp8_flow.cu"]
HEADERS = ["coat_device.cuh", "coat_internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "coat.h"),
                                                                 __file__]
    if not force and not _stale(lib, deps):
        return lib
    objdir = os.path.join(HERE, "_build_checked" if checked else "_build")
    os.makedirs(objdir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if ptxas_verbose else []) + (["-DCOAT_DEBUG"] if checked else [])

    def compile_one(src):
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        cmd = [nvcc()] + ARCH + NVCC_FLAGS + extra + ["-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
        if ptxas_verbose:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv,
                checked="--checked" in sys.argv))
