"""Build libebl.so (the CUDA library behind include/ebl.h) in-tree for sm_100a.

    python -m expert_bias_load_b200.build [--force] [--verbose] [--jobs N]

nvcc compiles every csrc/*.cu for sm_100a only, one object per source file and
several files at a time, and links them into expert_bias_load_b200/libebl.so
with the CUDA runtime linked statically, so the library loads without a CUDA
toolkit on the library path.  Objects go to _build/ at the repository root.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libebl.so")
ROOT = os.path.dirname(HERE)
OBJ_DIR = os.path.join(ROOT, "_build", "ebl")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC"]
LINK_FLAGS = [*ARCH, "-shared", "-cudart", "static"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    files = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files.append(os.path.join(ROOT, "include", "ebl.h"))
    return files


def _inputs():
    return sources() + _headers()


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _compile(nvcc, src, obj, verbose):
    cmd = [nvcc, *COMPILE_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", "-o", obj, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.stdout:
        sys.stderr.write(r.stdout)
    if r.stderr:
        sys.stderr.write(r.stderr)
    if r.returncode != 0:
        raise subprocess.CalledProcessError(r.returncode, cmd)
    return obj


def build(force: bool = False, verbose: bool = False, jobs: int = 0) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = nvcc_path()
    os.makedirs(OBJ_DIR, exist_ok=True)
    srcs = sources()
    objs = [os.path.join(OBJ_DIR, os.path.splitext(os.path.basename(s))[0] + ".o") for s in srcs]
    jobs = jobs or min(len(srcs), max(1, os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        list(pool.map(lambda so: _compile(nvcc, so[0], so[1], verbose), zip(srcs, objs)))
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call([nvcc, *LINK_FLAGS, "-o", tmp, *objs])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, jobs=a.jobs))
