"""Build the CUDA library ``libgated_delta.so`` in-tree (sm_100a).

    python -m gated_delta_rule_87_b200.build [--force] [--no-checked]

nvcc cross-compiles for sm_100a without a GPU.  The library links the CUDA
runtime statically and needs no libcuda at link time.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgated_delta.so")
BUILD_DIR = os.path.join(PKG, "_build")
# the same sources with every kernel-computed global index checked (sanitizer substitute)
LIB_CHECKED = os.path.join(PKG, "libgated_delta_checked.so")
BUILD_DIR_CHECKED = os.path.join(PKG, "_build_checked")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", 
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _build_variant(lib_path: str, build_dir: str, defines, force: bool, verbose: bool) -> str:
    os.makedirs(build_dir, exist_ok=True)
    objs = []
    procs = []
    hdrs = headers()
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src).replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [src] + hdrs):
            cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *defines, "-I", INCLUDE, "-I", CSRC, "-c", src,
                   "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE,
                                                stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out.strip() and (verbose or p.returncode):
            sys.stderr.write(out)
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(os.path.basename(f) for f in failed))
    if force or procs or _stale(lib_path, objs):
        tmp = lib_path + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib_path)
    return lib_path


def build(force: bool = False, verbose: bool = False, checked: bool = True) -> str:
    """Build ``libgated_delta.so`` and (unless ``checked`` is False) the
    bounds-checked ``libgated_delta_checked.so`` from the same sources."""
    _build_variant(LIB, BUILD_DIR, [], force, verbose)
    if checked:
        _build_variant(LIB_CHECKED, BUILD_DIR_CHECKED, ["-DGDR_BOUNDS_CHECK"], force, verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv,
          checked="--no-checked" not in sys.argv)
    print(LIB)
