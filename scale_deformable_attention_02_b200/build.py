"""Build the CUDA libraries in-tree, next to this file:

  libmsda.so          the product (include/msda.h, include/msda_debug.h);
  libmsda_checked.so  the same sources with -DMSDA_CHECKED: every value-map
                      access bounds-checked on the device (include/msda_checked.h).

nvcc cross-compiles for sm_100a without a GPU, so this runs anywhere the CUDA
toolkit is installed.  Objects go to _build/ and _build_checked/ next to this
file; a library is rebuilt only when a source or header is newer than it.

    python -m scale_deformable_attention_02_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
BUILD_CHECKED = os.path.join(PKG, "_build_checked")
LIB_PATH = os.path.join(PKG, "libmsda.so")
LIB_CHECKED_PATH = os.path.join(PKG, "libmsda_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmsda.so")
    return path


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def headers() -> list[str]:
    return (glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, obj: str, extra: list[str]) -> None:
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip() and "-v" in " ".join(extra):
        print(r.stderr)


def _build_one(lib_path: str, build_dir: str, defines: list[str], force: bool,
               verbose_ptxas: bool, ex: cf.Executor) -> list:
    os.makedirs(build_dir, exist_ok=True)
    hdrs = headers()
    extra = defines + (["-Xptxas", "-v"] if verbose_ptxas else [])
    objs, futs = [], []
    for s in sources():
        obj = os.path.join(build_dir, os.path.basename(s) + ".o")
        objs.append(obj)
        if force or verbose_ptxas or _stale(obj, [s, *hdrs]):
            futs.append(ex.submit(_compile, s, obj, extra))
    return [lib_path, objs, futs, force or bool(futs)]


def _link(lib_path: str, objs: list[str], relink: bool) -> None:
    if relink or _stale(lib_path, objs):
        tmp = lib_path + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib_path)


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = True) -> str:
    """Compile every CUDA/C++ source for sm_100a and link libmsda.so (and,
    unless checked=False, libmsda_checked.so).  Returns libmsda.so's path."""
    with cf.ThreadPoolExecutor(max_workers=8) as ex:
        jobs = [_build_one(LIB_PATH, BUILD, [], force, verbose_ptxas, ex)]
        if checked:
            jobs.append(_build_one(LIB_CHECKED_PATH, BUILD_CHECKED, ["-DMSDA_CHECKED"], force,
                                   False, ex))
        for lib_path, objs, futs, relink in jobs:
            for f in futs:
                f.result()
            _link(lib_path, objs, relink)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
