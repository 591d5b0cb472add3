"""Build libgla.so in-tree with nvcc for sm_100a.

    python -m chunkwise_linear_rnn_gla_b200.build [--force] [--verbose] [--checks]

--checks builds the checking library libgla_checks.so instead (-DGLA_CHECKS: every call runs the
checks of GLA_FLAG_CHECKS); the binding loads it when the environment sets GLA_CHECKS=1.

The library is a plain shared object (C ABI, no torch or Python types in its
signatures); the binding in this package loads it with ctypes.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libgla.so")
LIB_CHECKS = os.path.join(HERE, "libgla_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "gla.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(cmd):
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, verbose: bool = False, extra=None, checks: bool = False) -> str:
    """Compile every .cu under csrc/ into libgla.so (libgla_checks.so with checks=True; no-op when up
    to date). Each translation unit is compiled on its own, in parallel, into an object file under
    _build/ (no device code crosses translation units), then the objects are linked into the shared
    library."""
    lib = LIB_CHECKS if checks else LIB
    if not force and up_to_date(lib):
        return lib
    from concurrent.futures import ThreadPoolExecutor

    objdir = os.path.join(ROOT, "_build", "libgla_checks" if checks else "libgla")
    os.makedirs(objdir, exist_ok=True)
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
             "-I", os.path.join(ROOT, "include"), *(["-Xptxas", "-v"] if verbose else []), *(extra or []),
             *(["-DGLA_CHECKS"] if checks else [])]
    objs, cmds = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        cmds.append([nvcc(), *flags, "-c", src, "-o", obj])
    with ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 4)) as ex:
        results = list(ex.map(_compile, cmds))
    for r in results:
        if r.returncode != 0 or verbose:
            sys.stderr.write(r.stdout + r.stderr)
    if any(r.returncode != 0 for r in results):
        raise RuntimeError("nvcc failed building libgla.so")
    tmp = lib + ".tmp.%d" % os.getpid()
    r = subprocess.run([nvcc(), *ARCH, "-shared", *objs, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed linking " + os.path.basename(lib))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checks="--checks" in sys.argv))
