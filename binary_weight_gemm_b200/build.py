"""Build libobgemm.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m binary_weight_gemm_b200.build [--force] [--verbose] [--debug-bounds]``.
Each ``csrc/*.cu`` compiles to an object under ``_build/`` (in parallel), and
the objects link into ``binary_weight_gemm_b200/libobgemm.so`` with the CUDA
runtime linked statically.  A source hash stored beside the library skips the
build when nothing changed.

``--debug-bounds`` (or the environment variable ``OB_DEBUG_BOUNDS=1`` when ``build()``
is called without the argument) compiles with ``-DOB_DEBUG_BOUNDS``: kernels that
support it check every index they form against their buffers' lengths on the device
and record ``OB_ERR_DEVICE_BOUNDS`` instead of touching memory outside them.  It is a
checking build for tests, slower than the default one.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libobgemm.so")
STAMP = LIB + ".srchash"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libobgemm")
    return path


def _sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _flags(debug_bounds: bool) -> list[str]:
    return CFLAGS + (["-DOB_DEBUG_BOUNDS"] if debug_bounds else [])


def _debug_from_env() -> bool:
    return os.environ.get("OB_DEBUG_BOUNDS", "") not in ("", "0")


def _hash_inputs(debug_bounds: bool) -> str:
    h = hashlib.sha256()
    files = _sources() + sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                                if f.endswith((".cuh", ".h")))
    files.append(os.path.join(INCLUDE, "obgemm.h"))
    for f in files:
        h.update(f.encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(ARCH + _flags(debug_bounds)).encode())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          debug_bounds: bool | None = None) -> str:
    """Compile and link the library if its sources or flags changed; return its path."""
    if debug_bounds is None:
        debug_bounds = _debug_from_env()
    flags = _flags(debug_bounds)
    digest = _hash_inputs(debug_bounds)
    if not force and os.path.exists(LIB) and os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() == digest:
                return LIB
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()

    def compile_one(src: str) -> tuple[str, str]:
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
        cmd = [cc, *ARCH, *flags, "-c", src, "-o", obj]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{p.stdout}\n{p.stderr}")
        return obj, p.stdout + p.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, _sources()))
    if verbose or ptxas_verbose:
        for obj, log in results:
            if log.strip():
                print(f"--- {os.path.basename(obj)}\n{log}", file=sys.stderr)
    objs = [o for o, _ in results]
    tmp = LIB + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs]
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"link failed:\n{p.stdout}\n{p.stderr}")
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(digest)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true", help="print register/spill/smem use per kernel")
    ap.add_argument("--debug-bounds", action="store_true", help="device-side index checks (-DOB_DEBUG_BOUNDS)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_verbose=a.ptxas_verbose,
                debug_bounds=True if a.debug_bounds else None))
