"""Build libflux.so in-tree with nvcc for sm_100a (B200).

Each ``csrc/*.cu`` compiles to ``_build/<name>.o`` (skipped when up to date) and the
objects link into ``sparse_attention_layer_b200/lib/libflux.so``; with ``checked`` the
same sources compile with FLUX_CHECKED (bounds guards, include/flux.h) into
``_build/checked/`` and ``lib/libflux_checked.so``.  The CUDA runtime is
linked statically; the driver's tensor-map encoder is looked up at run time, so the
library loads on a machine without a GPU (only its compute calls need one).

Usage:  python -m sparse_attention_layer_b200.build [--force] [--verbose] [--checked]
"""

from __future__ import annotations

import argparse
import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_DIR = os.path.join(PKG, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libflux.so")
CHECKED_LIB_PATH = os.path.join(LIB_DIR, "libflux_checked.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH_FLAGS + [
    "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; libflux needs the CUDA toolkit to build")


def _deps() -> list:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "flux.h")]


def _stale(target: str, sources: list) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _compile(src: str, verbose: bool, checked: bool = False) -> str:
    obj_dir = os.path.join(BUILD_DIR, "checked") if checked else BUILD_DIR
    obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
    if _stale(obj, [src] + _deps()):
        cmd = [nvcc_path()] + NVCC_FLAGS + (["-DFLUX_CHECKED"] if checked else []) + \
            (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{res.stderr}")
        if verbose and res.stderr:
            sys.stderr.write(res.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile every kernel file and link libflux.so (libflux_checked.so with
    ``checked``); returns the library path."""
    obj_dir = os.path.join(BUILD_DIR, "checked") if checked else BUILD_DIR
    lib_path = CHECKED_LIB_PATH if checked else LIB_PATH
    os.makedirs(obj_dir, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if force:
        for s in sources:
            obj = os.path.join(obj_dir, os.path.basename(s)[:-3] + ".o")
            if os.path.exists(obj):
                os.remove(obj)
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(sources)) as pool:
        objs = list(pool.map(lambda s: _compile(s, verbose, checked), sources))
    if force or _stale(lib_path, objs):
        cmd = [nvcc_path()] + ARCH_FLAGS + ["-shared", "-o", lib_path] + objs
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link of {os.path.basename(lib_path)} failed:\n{res.stderr}")
    return lib_path


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="the bounds-guarded build")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, checked=args.checked))


if __name__ == "__main__":
    main()
