"""Build the in-tree CUDA library (libssm_scan.so) for sm_100a with nvcc.

The library is a plain C-ABI shared object (no torch types in its signatures):
cudart is linked statically and the driver entry point for TMA tensor maps is
looked up at run time, so the .so loads on machines without a GPU driver.

Each kernel family is its own translation unit (csrc/*.cu); they are compiled to
objects in parallel (csrc/_build/) and linked into one library.  An object is
rebuilt when its source or any header it includes (transitively) is newer.
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(CSRC, "_build")
LIB = os.path.join(HERE, "libssm_scan.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-warn-spills"]
LINK_FLAGS = [*ARCH, "-shared", "-cudart", "static"]

_INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def units():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps(path, seen=None):
    """The file and every local header it includes, transitively."""
    seen = set() if seen is None else seen
    path = os.path.normpath(path)
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    for inc in _INCLUDE.findall(open(path, encoding="utf-8").read()):
        _deps(os.path.join(os.path.dirname(path), inc), seen)
    return seen


def sources():
    """Every file the library is built from."""
    out = set()
    for u in units():
        out |= _deps(u)
    return sorted(out)


def _obj(unit):
    return os.path.join(OBJ, os.path.basename(unit)[:-3] + ".o")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def stale() -> bool:
    return _stale(LIB, sources())


def _compile(unit, extra, verbose):
    obj = _obj(unit)
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [NVCC, *COMPILE_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", unit, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(unit)}:\n{r.stdout}{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), jobs: int | None = None) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    todo = [u for u in units() if force or _stale(_obj(u), _deps(u))]
    jobs = jobs or max(1, min(len(todo), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=jobs) as ex:
        list(ex.map(lambda u: _compile(u, list(extra), verbose), todo))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *LINK_FLAGS, "-o", tmp, *[_obj(u) for u in units()]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    print(LIB)
