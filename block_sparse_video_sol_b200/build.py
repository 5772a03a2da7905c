"""Build step: compile the CUDA sources under csrc/ into the in-tree libsol.so.

Run as ``python -m block_sparse_video_sol_b200.build`` (or through
``__graft_entry__.build()``).  Every source is compiled for sm_100a only;
objects go to ``_build/`` and the shared library (static CUDA runtime) lands
next to this file, where the binding loads it.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libsol.so")
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsol.so")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "sol.h"), os.path.abspath(__file__)]


FAULT_OUT = os.path.join(PKG, "libsol_fault.so")


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, trace: bool = False,
          fault_test: bool = False) -> str:
    """Compile csrc/*.cu for sm_100a and link libsol.so; returns its path.

    ``trace`` builds a separate libsol_trace.so with the attention kernel's
    phase trace compiled in (for pipeline analysis; not used by the product).
    ``fault_test`` builds libsol_fault.so (SOL_FAULT_TEST: short wait limits
    and the withheld-arrive hook of sol_debug_drop_arrive), which the tests of
    the device-side timeout path load in a child process.
    """
    out = os.path.join(PKG, "libsol_trace.so") if trace else FAULT_OUT if fault_test else OUT
    if not force and not trace and up_to_date(out):
        return out
    nvcc = _nvcc()
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    if trace:
        extra.append("-DSOL_TRACE")
        if os.environ.get("SOL_TRACE_WARP"):
            extra.append("-DSOL_TRACE_WARP=" + os.environ["SOL_TRACE_WARP"])
    if fault_test:
        extra.append("-DSOL_FAULT_TEST")
    suffix = ".trace.o" if trace else ".fault.o" if fault_test else ".o"

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + suffix)
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with cf.ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose or ptxas_info:
        for obj, log in results:
            if log.strip():
                print(f"== {os.path.basename(obj)}\n{log}", file=sys.stderr)
    tmp = out + ".tmp"
    # --no-undefined: a symbol missing from the sources fails the build, not the first dlopen
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *[o for o, _ in results], "-cudart=static",
           "-Xlinker", "--no-undefined"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv,
                trace="--trace" in sys.argv, fault_test="--fault-test" in sys.argv))
