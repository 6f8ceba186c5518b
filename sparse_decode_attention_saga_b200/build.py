"""Builds ``libsaga.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m sparse_decode_attention_saga_b200.build [--force] [--verbose] [--debug]

Each ``csrc/*.cu`` file is compiled to an object under ``_build/`` (in
parallel), then linked into ``sparse_decode_attention_saga_b200/libsaga.so``.
Objects are rebuilt when their source or any header is newer.  ``--debug``
builds ``libsaga_debug.so`` instead (objects under ``_build/debug/``), with
SAGA_DEBUG defined: every position, count and slot a kernel reads from
another kernel's output is bounds-checked, an out-of-range one sets a sticky
error bit and is skipped.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIBRARY = os.path.join(PKG, "libsaga.so")
DEBUG_LIBRARY = os.path.join(PKG, "libsaga_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsaga.so")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    nvcc = _nvcc()
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    library = DEBUG_LIBRARY if debug else LIBRARY
    if debug:
        extra_flags = tuple(extra_flags) + ("-DSAGA_DEBUG=1",)
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    objects, jobs = [], []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objects.append(obj)
        if force or not os.path.exists(obj) or \
                os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header):
            cmd = [nvcc] + NVCC_FLAGS + list(extra_flags) + ["-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    failed = []
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose or r.returncode:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode:
                failed.append(cmd[-3])
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    if jobs or force or not os.path.exists(library):
        tmp = library + ".tmp"
        cmd = [nvcc] + ARCH + ["-shared", "-o", tmp] + objects
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
        os.replace(tmp, library)
    return library


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))
