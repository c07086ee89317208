"""Build libpkm.so (the PKM CUDA library) in-tree with nvcc for sm_100a.

    python product_key_memory_b200/build.py   # run as a script: importing the
                                              # package needs the built library

Every .cu file under csrc/ is compiled with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` and linked into one
shared library with the CUDA runtime linked statically, so the library loads
beside any PyTorch build.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libpkm.so")
BUILD_DIR = os.path.join(ROOT, "_build")
# Test build: every pipeline wait of the tensor-core kernels gives up as soon as it is
# not satisfied within one try (a 1 ns limit; the drains keep their full second), so
# the first wait on a copy from HBM always runs out and tests exercise the timeout
# path; see tests/test_timeout_gpu.py. Loaded only through PKM_LIBRARY.
WAITTEST_LIB = os.path.join(HERE, "libpkm_waittest.so")
WAITTEST_DEFINES = ("-DPKM_WAIT_LIMIT_NS=1ull", "-DPKM_TRY_WAIT_HINT_NS=100")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    deps = [src] + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(d) > os.path.getmtime(obj) for d in deps)


def build(verbose: bool = False, force: bool = False, extra=(), lib: str = LIB,
          build_dir: str = BUILD_DIR) -> str:
    os.makedirs(build_dir, exist_ok=True)
    objs = []
    procs = []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _stale(obj, src):
            cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                                stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if p.returncode != 0:
            failed.append((src, out))
        elif verbose and out.strip():
            print(out, flush=True)
    if failed:
        msg = "\n".join("%s:\n%s" % (s, o) for s, o in failed)
        raise RuntimeError("nvcc failed:\n" + msg)
    if force or procs or not os.path.exists(lib):
        tmp = lib + ".tmp%d" % os.getpid()
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        subprocess.check_call(cmd)
        os.replace(tmp, lib)
    return lib


def build_waittest(verbose: bool = False, force: bool = False) -> str:
    return build(verbose, force, extra=WAITTEST_DEFINES, lib=WAITTEST_LIB,
                 build_dir=os.path.join(BUILD_DIR, "waittest"))


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv,
          extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ())
    print(LIB)
    if "--no-waittest" not in sys.argv:
        print(build_waittest(verbose=False, force="--force" in sys.argv))
