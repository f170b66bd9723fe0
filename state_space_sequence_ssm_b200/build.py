"""Build the in-tree CUDA library ``libm3.so`` for sm_100a with nvcc, and its
bounds build ``libm3_bounds.so`` (every kernel compiled with M3_DEVICE_CHECKS:
device-side index checks that record a failure instead of trapping).

Usage: ``python -m state_space_sequence_ssm_b200.build [--force] [--verbose]
[--bounds]``.  Objects go to ``state_space_sequence_ssm_b200/_build/`` (the
bounds build's to ``_build/bounds/``); the shared libraries land next to this
file so that they travel with the source tree.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libm3.so")
BOUNDS_LIB = os.path.join(HERE, "libm3_bounds.so")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    return (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build(force: bool = False, verbose: bool = False, extra_flags=None, bounds: bool = False) -> str:
    """Compile and link one library: libm3.so, or with ``bounds`` libm3_bounds.so."""
    obj_dir = os.path.join(OBJ, "bounds") if bounds else OBJ
    lib = BOUNDS_LIB if bounds else LIB
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))
    deps = _deps()
    flags = NVCC_FLAGS + (["-DM3_DEVICE_CHECKS"] if bounds else []) + list(extra_flags or [])
    jobs = []
    for s in srcs:
        o = os.path.join(obj_dir, os.path.basename(s) + ".o")
        if force or _stale(o, [s] + deps):
            jobs.append((s, o))

    def compile_one(job):
        s, o = job
        cmd = [nvcc()] + ARCH + flags + ["-c", s, "-o", o]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(s)}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        return o

    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(compile_one, jobs))
    objs = [os.path.join(obj_dir, os.path.basename(s) + ".o") for s in srcs]
    if force or jobs or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    return lib


def build_all(force: bool = False, verbose: bool = False) -> None:
    """Both libraries, compiled side by side."""
    with ThreadPoolExecutor(max_workers=2) as ex:
        for f in [ex.submit(build, force, verbose, None, b) for b in (False, True)]:
            f.result()


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register/smem usage")
    ap.add_argument("--bounds", action="store_true", help="the bounds build (device index checks)")
    a = ap.parse_args()
    print(build(force=a.force or a.ptxas_v, verbose=a.verbose or a.ptxas_v,
                extra_flags=["-Xptxas", "-v"] if a.ptxas_v else None, bounds=a.bounds))
