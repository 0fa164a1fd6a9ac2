"""Builds libprism.so (the C-ABI CUDA library) in-tree for sm_100a.

Each .cu under csrc/ is compiled with nvcc to an object, then linked into
``dynamic_block_sparse_shape_b200/libprism.so`` with the CUDA runtime linked
statically, so the library loads without a GPU and depends only on the driver
at run time. ``python -m dynamic_block_sparse_shape_b200.build`` runs it.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
OUT = os.path.join(HERE, "libprism.so")
OBJ_DIR = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


# Test-only variant: device waits give up after 50 ms instead of about 2 s, and the
# forward's copy producer can be told (through a workspace word) to skip one step's
# copies, so that a test can make a bounded wait run out and check the reported status.
FAULT_INJECTION_FLAGS = ["-DPRISM_FAULT_INJECTION", "-DPRISM_WAIT_LIMIT_NS=50000000ull"]


def variant_path(tag: str) -> str:
    return os.path.join(HERE, f"libprism_{tag}.so")


def build_variant(tag: str, flags, verbose: bool = False) -> str:
    """Builds a separately named copy of the library with extra compile flags
    (objects in _build_<tag>/, library libprism_<tag>.so); returns its path."""
    return build(verbose=verbose, extra_flags=flags, obj_dir=os.path.join(HERE, f"_build_{tag}"),
                 out=variant_path(tag))


def build(verbose: bool = False, force: bool = False, extra_flags=None, obj_dir=None, out=None) -> str:
    """Compile every .cu for sm_100a and link libprism.so; returns its path."""
    obj_dir = obj_dir or OBJ_DIR
    out = out or OUT
    os.makedirs(obj_dir, exist_ok=True)
    srcs = _sources()
    hdrs = _headers()
    flags = FLAGS + list(extra_flags or [])
    objs = []
    jobs = []
    for s in srcs:
        o = os.path.join(obj_dir, os.path.splitext(os.path.basename(s))[0] + ".o")
        objs.append(o)
        if force or _stale(o, [s] + hdrs + [__file__]):
            jobs.append([nvcc(), *ARCH, *flags, "-c", s, "-o", o])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, file=sys.stderr)

    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or _stale(out, objs):
        tmp = out + ".tmp"
        run([nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs])
        os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
