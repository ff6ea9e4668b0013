"""Builds libbitnet_b200.so (the CUDA library behind include/bitnet.h) in-tree.

    python -m bitlinear_absmean_ternary_b200.build [--force]

nvcc cross-compiles for sm_100a only; no GPU is needed to build.  Every .cu
file under csrc/ is one translation unit (a kernel family with its entry
points); they compile in parallel into csrc/_build/ and link into one shared
library.  A unit is rebuilt when it or any header it includes is newer than
its object.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbitnet_b200.so")
OBJDIR = os.path.join(CSRC, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-warn-spills"]


def units() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def sources() -> list:
    return sorted(units() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def _deps(path: str, seen=None) -> set:
    """The file and every quoted include it reaches (csrc/ and include/)."""
    seen = set() if seen is None else seen
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    with open(path, encoding="utf-8") as f:
        for name in re.findall(r'#include\s+"([^"]+)"', f.read()):
            for d in (os.path.dirname(path), CSRC, INCLUDE):
                p = os.path.join(d, name)
                if os.path.exists(p):
                    _deps(p, seen)
                    break
    return seen


def _obj(unit: str) -> str:
    return os.path.join(OBJDIR, os.path.basename(unit)[:-3] + ".o")


def _stale_obj(unit: str) -> bool:
    o = _obj(unit)
    if not os.path.exists(o):
        return True
    t = os.path.getmtime(o)
    return any(os.path.getmtime(d) > t for d in _deps(unit))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def _compile(unit: str, extra: list, verbose: bool) -> str:
    o = _obj(unit)
    tmp = o + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I" + INCLUDE, "-I" + CSRC, "-c", unit, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(unit)}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout.strip() or r.stderr.strip()):
        print(r.stdout + r.stderr, flush=True)
    os.replace(tmp, o)
    return o


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    """Compile the stale units in parallel and link the library; returns its path."""
    if not force and not stale():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    todo = [u for u in units() if force or _stale_obj(u)]
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(todo) or 1, os.cpu_count() or 1))) as ex:
        list(ex.map(lambda u: _compile(u, list(extra_flags or []), verbose), todo))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *[_obj(u) for u in units()]]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
