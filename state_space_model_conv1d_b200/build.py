"""Build ``libssm.so`` in-tree from ``csrc/*.cu`` for sm_100a with nvcc.

Each translation unit is compiled to an object in ``_build/`` (in parallel,
only when its sources changed) and linked into
``state_space_model_conv1d_b200/libssm.so`` with the CUDA runtime linked
statically, so the library needs nothing from PyTorch.

``build(check_bounds=True)`` (``--check-bounds``) builds the bounds-checked
variant ``libssm_checked.so`` instead: every source with ``SSM_CHECK_BOUNDS``
defined and relocatable device code (the kernels of every translation unit
record into one device-wide bounds record), objects in ``_build_checked/``.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libssm.so")
BUILD_CHECKED = os.path.join(ROOT, "_build_checked")
LIB_CHECKED = os.path.join(PKG, "libssm_checked.so")
CHECKED_FLAGS = ["-DSSM_CHECK_BOUNDS", "-rdc=true"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fvisibility=hidden"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def _compile(src: str, verbose: bool, checked: bool = False) -> str:
    obj = os.path.join(BUILD_CHECKED if checked else BUILD, os.path.basename(src)[:-3] + ".o")
    newest = max([os.path.getmtime(src)] + [os.path.getmtime(h) for h in _headers()])
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *(CHECKED_FLAGS if checked else []), "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose: bool = False, check_bounds: bool = False) -> str:
    out_dir, lib = (BUILD_CHECKED, LIB_CHECKED) if check_bounds else (BUILD, LIB)
    os.makedirs(out_dir, exist_ok=True)
    srcs = _sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, check_bounds), srcs))
    if os.path.exists(lib) and os.path.getmtime(lib) >= max(os.path.getmtime(o) for o in objs):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", *(["-rdc=true"] if check_bounds else []), "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, check_bounds="--check-bounds" in sys.argv))
