"""Build libcql.so in-tree with nvcc for sm_100a.

    python -m sparse_quantized_rank_b200.build          # build if stale
    python -m sparse_quantized_rank_b200.build --force  # always rebuild
    python -m sparse_quantized_rank_b200.build --checked  # libcql_checked.so

The checked variant is compiled with -DCQL_CHECKED: every plane read,
activation read, workspace access and output store of the forward kernels
is range-checked, and an index outside its buffer records CQL_ERR_RANGE in
the device error word (the access is skipped) instead of touching memory.
It stands in for a memory checker on machines where none can run.

The library is compiled straight from ``csrc/*.cu`` with
``-gencode arch=compute_100a,code=sm_100a`` (B200 only) and the CUDA runtime
linked statically, so the shared object depends on nothing but the driver.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libcql.so")
LIB_CHECKED = os.path.join(HERE, "libcql_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put CUDA 12.8+ on PATH)")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile every CUDA source into libcql.so (libcql_checked.so with
    checked=True) next to this file; return its path."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = _nvcc()
    objdir = os.path.join(HERE, "_build_checked" if checked else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    extra = ["-DCQL_CHECKED"] if checked else []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr, file=sys.stderr)
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", *objs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="the range-checked variant")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, checked=a.checked))
