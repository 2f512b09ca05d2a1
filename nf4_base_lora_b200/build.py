"""Build libnf4lora.so in-tree with nvcc for sm_100a.

    python nf4_base_lora_b200/build.py [--force] [--debug]

Each .cu under csrc/ is compiled to an object in parallel (relocatable device
code, so the kernels share one device status word), then device-linked into
``nf4_base_lora_b200/lib/libnf4lora.so``.  No GPU is needed to build.

``--debug`` builds ``lib/libnf4lora_debug.so`` with NF4LORA_DEBUG defined: the
kernels then check the index and alignment of their memory accesses and
record the first failed check instead of faulting (see nf4lora_debug_site in
include/nf4lora.h).  The binding loads it when NF4LORA_DEBUG=1 is set.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "lib")
BUILD_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libnf4lora.so")
DEBUG_LIB = os.path.join(OUT_DIR, "libnf4lora_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-rdc=true", "-Xcompiler", "-fPIC",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found")
    return exe


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, extra, build_dir: str = BUILD_DIR) -> str:
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    if _stale(obj, [src] + _headers()):
        cmd = [nvcc()] + ARCH + FLAGS + list(extra) + ["-c", src, "-o", obj]
        subprocess.run(cmd, check=True)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    build_dir = BUILD_DIR + ("_debug" if debug else "")
    os.makedirs(OUT_DIR, exist_ok=True)
    os.makedirs(build_dir, exist_ok=True)
    srcs = _sources()
    if force:
        for o in glob.glob(os.path.join(build_dir, "*.o")):
            os.remove(o)
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DNF4LORA_DEBUG"] if debug else [])
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, build_dir), srcs))
    if force or _stale(lib, objs):
        tmp = lib + ".tmp%d" % os.getpid()
        cmd = [nvcc()] + ARCH + ["-shared", "-rdc=true", "-Xcompiler", "-fPIC", "-o", tmp] + objs
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas-v" in sys.argv, debug="--debug" in sys.argv))
