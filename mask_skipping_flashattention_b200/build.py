"""Build ``libbfa.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python mask_skipping_flashattention_b200/build.py [--force] [--verbose]`` (run by path:
importing the package would load the library being rebuilt).
Objects go to ``_build/`` at the repository root; the shared library is written
next to this file so that it travels with the source tree.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libbfa.so")
LIB_CHECKED = os.path.join(PKG, "libbfa_checked.so")
SOURCES = ["planner.cu", "fwd.cu", "bwd.cu", "bfa_host.cu"]
HEADERS = ["ptx.cuh", "plan_types.cuh", "fwd_params.cuh", "pred.cuh", "tile_mask.cuh", "bwd_params.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-Xptxas", "-v",
         f"-I{os.path.join(ROOT, 'include')}"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libbfa.so")


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    """Build libbfa.so and its bounds-checked twin libbfa_checked.so (-DBFA_CHECKED)."""
    lib = _build_one(LIB, BUILD, [], force, verbose)
    _build_one(LIB_CHECKED, os.path.join(BUILD, "checked"), ["-DBFA_CHECKED"], force, verbose)
    return lib


def _build_one(lib_path, build_dir, defines, force, verbose):
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "bfa.h")]
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            cmd = [nvcc, *ARCH, *FLAGS, *defines, "-c", s, "-o", o]
            r = subprocess.run(cmd, capture_output=True, text=True)
            log = r.stdout + r.stderr
            with open(o + ".log", "w") as f:
                f.write(" ".join(cmd) + "\n" + log)
            if r.returncode != 0:
                sys.stderr.write(log)
                raise RuntimeError(f"nvcc failed on {src}")
            if verbose:
                sys.stdout.write(log)
    if force or _stale(lib_path, objs):
        cmd = [nvcc, *ARCH, "-shared", "-o", lib_path, *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"link of {os.path.basename(lib_path)} failed")
    return lib_path


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
