"""Build the CUDA libraries (sm_100a) in-tree with nvcc.

libmoe.so is the product.  libmoe_debug.so is the same sources compiled with
MOE_DEBUG: its kernels also check the indices they read from their inputs
(expert ids, expert offsets, permuted rows) and report a violation through the
workspace error word (moe_device_status -> MOE_ERR_DEVICE_BOUNDS) instead of
making the access.  Each csrc/*.cu is compiled to an object under _build/ (in
parallel), then linked with the static CUDA runtime.
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
OUT = os.path.join(PKG, "libmoe.so")
OUT_DEBUG = os.path.join(PKG, "libmoe_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*"))) + [os.path.join(ROOT, "include", "moe.h")]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose, debug):
    obj = os.path.join(BUILD, os.path.basename(src) + (".debug.o" if debug else ".o"))
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DMOE_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def _link(objs, out):
    tmp = out + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Builds libmoe.so (and, with debug=True, libmoe_debug.so) when stale;
    returns the path of libmoe.so."""
    deps = _deps()
    targets = [(OUT, False)] + ([(OUT_DEBUG, True)] if debug else [])
    todo = [(out, dbg) for out, dbg in targets if force or verbose or _stale(out, deps)]
    if not todo:
        return OUT
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    jobs = [(src, dbg) for _, dbg in todo for src in srcs]
    with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
        results = list(ex.map(lambda j: _compile(j[0], verbose, j[1]), jobs))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    for out, dbg in todo:
        _link([o for (o, _), (_, d) in zip(results, jobs) if d == dbg], out)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
