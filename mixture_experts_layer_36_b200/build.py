"""Build libmoe.so in-tree with nvcc for sm_100a (no GPU needed to compile).

    python -m mixture_experts_layer_36_b200.build [--force] [--verbose-ptxas] [--checks]

--checks builds the library with MOE_CHECKS: extra device-side input checks
that report into the caller's status word (e.g. an expert listed twice for
one token).  It replaces the in-tree libmoe.so; build again without the flag
(with --force) to return to the normal library.
"""
import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [
        os.path.join(ROOT, "include", "moe.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, ptxas_verbose: bool = False, jobs: int = 8,
          checks: bool = False) -> str:
    if not force and not checks and up_to_date():
        return LIB
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = ["-O3", "-std=c++17", "-lineinfo", "-cudart", "shared", "-Xcompiler", "-fPIC",
             "-I", os.path.join(ROOT, "include"), *ARCH]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    if checks:
        flags += ["-DMOE_CHECKS"]
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append(subprocess.Popen([NVCC, *flags, "-c", src, "-o", obj]))
        if len(procs) >= jobs:
            _wait(procs)
            procs = []
    _wait(procs)
    tmp = LIB + f".{os.getpid()}.tmp"
    subprocess.check_call([NVCC, "-shared", "-cudart", "shared", *ARCH, "-o", tmp, *objs, "-ldl"])
    os.replace(tmp, LIB)
    return LIB


def _wait(procs):
    bad = [p for p in procs if p.wait() != 0]
    if bad:
        raise RuntimeError("nvcc failed")


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--checks", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas, checks=a.checks))
    sys.exit(0)
