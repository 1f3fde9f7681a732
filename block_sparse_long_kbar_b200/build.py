"""Build libsgqa.so in-tree for sm_100a with nvcc (object files compiled in parallel).

variant="checks" builds libsgqa_checks.so, the same sources with -DSGQA_CHECKS: the kernels test
the indices they compute from data against their buffers and record SGQA_ERR_DEVICE_CHECK
instead of making an out-of-range access (the debug build the tests run alongside the normal
one)."""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
SO = os.path.join(HERE, "libsgqa.so")
SO_CHECKS = os.path.join(HERE, "libsgqa_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
         "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + [
        os.path.join(ROOT, "include", "sgqa.h")]


def _variant(variant: str):
    if variant == "checks":
        return os.path.join(HERE, "_build_checks"), SO_CHECKS, ["-DSGQA_CHECKS"]
    if variant:
        raise ValueError(f"unknown library variant {variant!r}")
    return BUILD, SO, []


def needs_build(variant: str = "") -> bool:
    so = _variant(variant)[1]
    if not os.path.exists(so):
        return True
    t = os.path.getmtime(so)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force: bool = False, verbose: bool = False, extra=None, variant: str = "") -> str:
    build_dir, so, vflags = _variant(variant)
    if not force and not needs_build(variant):
        return so
    os.makedirs(build_dir, exist_ok=True)
    extra = vflags + list(extra or [])

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = ["nvcc", *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
        if verbose and r.stderr:
            print(r.stderr, file=sys.stderr)
        return obj

    with concurrent.futures.ThreadPoolExecutor(max_workers=8) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = so + ".tmp"
    cmd = ["nvcc", *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, so)
    return so


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else None,
                variant="checks" if "--checks" in sys.argv else ""))
