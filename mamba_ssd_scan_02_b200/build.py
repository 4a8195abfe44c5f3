"""Build libssd.so (the CUDA library behind include/ssd.h) in-tree for sm_100a.

    python -m mamba_ssd_scan_02_b200.build [--force] [-v] [--debug-bounds]

Each csrc/*.cu is compiled by nvcc to an object under _build/ (in parallel, skipped when
up to date) and linked into mamba_ssd_scan_02_b200/libssd.so against the shared CUDA
runtime, so that the process uses one runtime together with PyTorch.  With --debug-bounds the
same sources are compiled with -DSSD_DEBUG_BOUNDS (device-side index checks that latch
SSD_ERR_DEVICE_BOUNDS) into libssd_debug.so, for tests.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(ROOT, "_build", "obj")
LIB = os.path.join(PKG, "libssd.so")
OBJ_DEBUG = os.path.join(ROOT, "_build", "obj_debug")
LIB_DEBUG = os.path.join(PKG, "libssd_debug.so")
HEADERS = [os.path.join(ROOT, "include", "ssd.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                     "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libssd.so")
    return cand


def _cuda_lib_dir() -> str:
    nv = os.path.realpath(_nvcc())
    return os.path.join(os.path.dirname(os.path.dirname(nv)), "lib64")


def _newest(paths) -> float:
    return max(os.path.getmtime(p) for p in paths)


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          debug_bounds: bool = False) -> str:
    """Compile every csrc/*.cu and link libssd.so (or, with debug_bounds, libssd_debug.so with
    the device-side index checks); returns its path."""
    obj_dir, lib = (OBJ_DEBUG, LIB_DEBUG) if debug_bounds else (OBJ, LIB)
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = HEADERS + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
    hdr_time = _newest(hdrs)
    nvcc = _nvcc()
    flags = NVCC_FLAGS + (extra_flags or []) + (["-DSSD_DEBUG_BOUNDS"] if debug_bounds else [])

    def compile_one(src):
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        if (not force and os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
                and os.path.getmtime(obj) >= hdr_time):
            return obj, ""
        cmd = [nvcc, *flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, srcs))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            if log.strip():
                print(log)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < _newest(objs):
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "shared", "-o", lib, *objs,
               "-Xlinker", f"-rpath,{_cuda_lib_dir()}"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug_bounds=a.debug_bounds))
