"""Builds libvdn.so (sm_100a) in-tree from csrc/*.cu with nvcc, and the range-checked test
build libvdn_checked.so (VDN_BOUNDS_CHECK=1: the tensor-core kernels check every index they
derive from the layout tables; a stand-in for a device memory checker).

    python -m hybrid_softmax_linear_b200.build [--jobs N] [--verbose-ptxas] [--checked]

Objects go to _build/ (and _build/checked/) at the repository root; the shared libraries
land next to this file, where the Python binding loads them from.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libvdn.so")
OUT_CHECKED = os.path.join(PKG, "libvdn_checked.so")
BUILD = os.path.join(ROOT, "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, ptxas_v: bool, checked: bool = False) -> tuple[str, str]:
    bdir = os.path.join(BUILD, "checked") if checked else BUILD
    obj = os.path.join(bdir, os.path.basename(src) + ".o")
    deps = [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "vdn.h")]
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(x) for x in deps) and not ptxas_v:
        return obj, ""
    extra = ["-DVDN_BOUNDS_CHECK=1"] if checked else []
    cmd = [nvcc()] + ARCH + FLAGS + extra + (["-Xptxas", "-v"] if ptxas_v else []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
    return obj, r.stderr


def build(jobs: int | None = None, ptxas_v: bool = False, quiet: bool = True, checked: bool = False) -> str:
    """Compiles and links libvdn.so, or with checked=True the range-checked libvdn_checked.so."""
    os.makedirs(os.path.join(BUILD, "checked") if checked else BUILD, exist_ok=True)
    out = OUT_CHECKED if checked else OUT
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(jobs or min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, ptxas_v, checked), srcs))
    objs = [o for o, _ in results]
    if ptxas_v or not quiet:
        for _, log in results:
            if log:
                sys.stderr.write(log)
    newest = max(os.path.getmtime(o) for o in objs)
    if not os.path.exists(out) or os.path.getmtime(out) < newest:
        cmd = [nvcc()] + ARCH + ["-shared", "-o", out] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--checked", action="store_true", help="build the range-checked libvdn_checked.so")
    a = ap.parse_args()
    print(build(a.jobs, a.verbose_ptxas, quiet=False, checked=a.checked))
