"""Build the in-tree CUDA library ``libdg.so`` (sm_100a) and the oracle's nothing.

Usage: python -m discrete_text_diffusion_b200.build [--force] [--jobs N]

Each ``csrc/*.cu`` is compiled to an object with nvcc for
``-gencode arch=compute_100a,code=sm_100a`` and linked into one shared
library next to this file.  Objects are rebuilt when their source or any
header changed.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdg.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "dg.h")]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, extra):
    obj = os.path.join(OBJ, os.path.basename(src) + ".o")
    if not _stale(obj, [src] + _headers()) and not extra.get("force"):
        return obj, None
    cmd = [NVCC] + ARCH + FLAGS + extra.get("flags", []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        return obj, f"{' '.join(cmd)}\n{r.stdout}\n{r.stderr}"
    return obj, None


def build(force=False, jobs=None, verbose=False, extra_flags=None):
    """Compile every csrc/*.cu for sm_100a and link libdg.so.  Returns the path."""
    os.makedirs(OBJ, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    extra = {"force": force, "flags": list(extra_flags or [])}
    objs, errs = [], []
    with cf.ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
        for obj, err in ex.map(lambda s: _compile(s, extra), srcs):
            objs.append(obj)
            if err:
                errs.append(err)
    if errs:
        raise RuntimeError("nvcc failed:\n" + "\n\n".join(errs))
    if force or _stale(LIB, objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", LIB] + objs + ["-lcuda"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    if verbose:
        print(LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=None)
    ap.add_argument("--ptxas-v", action="store_true", help="print register / smem usage")
    args = ap.parse_args()
    flags = ["-Xptxas", "-v"] if args.ptxas_v else []
    try:
        build(force=args.force or args.ptxas_v, jobs=args.jobs, verbose=True, extra_flags=flags)
    except RuntimeError as e:
        print(e, file=sys.stderr)
        sys.exit(1)
