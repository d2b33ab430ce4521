"""Builds libisoq.so in-tree with nvcc for sm_100a (B200).

    python rotated_bit_kv_isoquant_b200/build.py [--force] [--checked]

(run as a script: importing the package itself needs the library)

Each .cu under csrc/ compiles to an object in parallel, then the objects link into
rotated_bit_kv_isoquant_b200/libisoq.so.  Needs only nvcc (no GPU).

--checked builds the bounds-checked variant libisoq_checked.so (-DISOQ_CHECK_BOUNDS, its
own object folder): every global, shared and tensor-memory index of the kernels is
compared with its extent, and a bad one skips the access and sets ISOQ_ST_BOUNDS in the
status word instead of faulting.  The same entry points; slower; for tests.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libisoq.so")
CHECKED_LIB = os.path.join(PKG, "libisoq_checked.so")
CHECKED_FLAGS = ["-DISOQ_CHECK_BOUNDS"]

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", f"-I{os.path.join(ROOT, 'include')}"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(), checked: bool = False) -> str:
    lib = CHECKED_LIB if checked else LIB
    if not force and up_to_date(lib):
        return lib
    build_dir = os.path.join(BUILD, "checked") if checked else BUILD
    flags = [*FLAGS, *(CHECKED_FLAGS if checked else []), *extra_flags]
    os.makedirs(build_dir, exist_ok=True)
    procs, objs = [], []
    for src in _sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *flags, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT),
                      src))
        objs.append(obj)
    failed = []
    for p, src in procs:
        out, _ = p.communicate()
        if out and (verbose or p.returncode):
            sys.stdout.write(out.decode())
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-lcudart"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv or "--verbose" in sys.argv,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [],
                checked="--checked" in sys.argv))
