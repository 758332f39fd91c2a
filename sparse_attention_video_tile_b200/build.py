"""Builds the in-tree CUDA library ``libsta.so`` for sm_100a with nvcc, and its
checked twin ``libsta_checked.so`` (device-side bounds checks on the forward
kernel's schedule-derived indices, for tests).

Usage: ``python -m sparse_attention_video_tile_b200.build [--verbose]``.
The library lands next to this file so the Python binding finds it; it is
rebuilt when a source is newer than the library.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libsta.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["api.cu", "attention.cu", "backward.cu", "noalloc.cu", "reorder.cu", "schedule.cpp"]
HEADERS = ["internal.h", "ptx.cuh"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libsta.so")
    return path


LIB_CHECKED = os.path.join(HERE, "libsta_checked.so")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "sta.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def _build_lib(lib: str, obj_dir: str, defines, verbose: bool) -> None:
    os.makedirs(obj_dir, exist_ok=True)
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(obj_dir, src + ".o")
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *defines, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose and src.endswith(".cu"):
            cmd += ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
        objs.append(obj)
    failed = []
    for src, pr in procs:
        out = pr.communicate()[0]
        if verbose or pr.returncode != 0:
            sys.stderr.write(out)
        if pr.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"linking {os.path.basename(lib)} failed")
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source and link libsta.so and its checked twin
    libsta_checked.so (device-side bounds checks, STA_DEVICE_CHECKS=1); returns
    the path of libsta.so."""
    if force or _stale(LIB):
        _build_lib(LIB, BUILD_DIR, [], verbose)
    if force or _stale(LIB_CHECKED):
        _build_lib(LIB_CHECKED, os.path.join(BUILD_DIR, "checked"), ["-DSTA_DEVICE_CHECKS=1"], verbose)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
