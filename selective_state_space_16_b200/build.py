"""Build the in-tree CUDA library (libssm_scan.so) for sm_100a with nvcc.

The library is a plain C-ABI shared object (no torch types in its signatures):
cudart is linked statically and the driver entry point for TMA tensor maps is
looked up at run time, so the .so loads on machines without a GPU driver.

Each kernel family is its own translation unit (csrc/*.cu); they are compiled to
objects in parallel (csrc/_build/) and linked into one library.  An object is
rebuilt when its source or any header it includes (transitively) is newer.

build(debug=True) makes libssm_scan_debug.so (objects in csrc/_build_debug/): the
same sources with -DSSM_DEBUG_CHECKS, whose kernels range-check their indices and
report SSM_ERR_BOUNDS through the workspace status word instead of faulting.
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
OBJ_DEBUG = os.path.join(CSRC, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libssm_scan_debug.so")
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


def _obj(unit, debug=False):
    return os.path.join(OBJ_DEBUG if debug else OBJ, os.path.basename(unit)[:-3] + ".o")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def stale(debug: bool = False) -> bool:
    return _stale(LIB_DEBUG if debug else LIB, sources())


def _compile(unit, extra, verbose, debug=False):
    obj = _obj(unit, debug)
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [NVCC, *COMPILE_FLAGS, *(["-DSSM_DEBUG_CHECKS"] if debug else []), *extra, "-I",
           os.path.join(ROOT, "include"), "-c", unit, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(unit)}:\n{r.stdout}{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), jobs: int | None = None, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not stale(debug):
        return lib
    os.makedirs(OBJ_DEBUG if debug else OBJ, exist_ok=True)
    todo = [u for u in units() if force or _stale(_obj(u, debug), _deps(u))]
    jobs = jobs or max(1, min(len(todo), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=jobs) as ex:
        list(ex.map(lambda u: _compile(u, list(extra), verbose, debug), todo))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *LINK_FLAGS, "-o", tmp, *[_obj(u, debug) for u in units()]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
