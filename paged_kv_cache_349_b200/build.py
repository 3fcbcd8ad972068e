"""Build step of the CUDA library: nvcc -> ``libpa.so`` next to this file.

Compiles every ``csrc/*.cu`` / ``csrc/*.cpp`` for sm_100a only
(``-gencode arch=compute_100a,code=sm_100a``), with the CUDA runtime linked
statically so the library needs nothing but the NVIDIA driver at run time.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libpa.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, verbose: bool = False, defines=(), out: str = None) -> str:
    """Compile the library if a source is newer than ``libpa.so``; return its path.

    ``defines`` (``NAME=VALUE`` strings) and ``out`` make a tuning build of the
    same sources at another path (always rebuilt); the package loads it when
    the environment names it in ``PA_LIBRARY``."""
    target = out or LIB
    if not out and not defines and not force and not _stale():
        return LIB
    tmp = target + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC,-O3", "-shared", "-cudart", "static", "-I", INCLUDE,
           *[f"-D{d}" for d in defines], "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libpa.so")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser(description="build libpa.so (sm_100a)")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", dest="verbose", action="store_true", help="print ptxas register and spill counts")
    ap.add_argument("--define", action="append", default=[], help="NAME=VALUE for a tuning build")
    ap.add_argument("--out", default=None, help="output path of a tuning build")
    a = ap.parse_args()
    if a.define and not a.out:
        ap.error("a tuning build (--define) needs --out, so the library itself is left as built")
    print(build(force=a.force, verbose=a.verbose, defines=a.define, out=a.out))
