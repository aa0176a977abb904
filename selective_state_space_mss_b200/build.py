"""Build libmss.so in-tree with nvcc for sm_100a.

    python -m selective_state_space_mss_b200.build [--force] [--ptxas-v]

Each translation unit of csrc/ (the C ABI in mss_api.cu, the forward-pass
launchers fwd_*.cu, the decode launchers decode.cu) is compiled to an object
in parallel, then the objects are linked against the static CUDA runtime so
that the library loads without any particular libcudart on the search path.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmss.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

OBJ_DIR = os.path.join(HERE, "_build")
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*")) + [os.path.join(ROOT, "include", "mss.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _sources())


def translation_units():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    tag = f"{os.getpid()}"

    def compile_one(src):
        obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + f".{tag}.o")
        cmd = [NVCC, *NVCC_FLAGS, *extra_flags, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, r

    units = translation_units()
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(units), os.cpu_count() or 1))) as ex:
        results = list(ex.map(compile_one, units))
    failed = [(src, r) for src, _, r in results if r.returncode != 0]
    for src, _, r in results:
        if r.stdout or r.stderr:
            sys.stdout.write(r.stdout)
            sys.stderr.write(r.stderr)
    if failed:
        raise subprocess.CalledProcessError(failed[0][1].returncode, f"nvcc {failed[0][0]}")
    objs = [obj for _, obj, _ in results]
    tmp = LIB + f".tmp{tag}"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    try:
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if os.path.exists(obj):
                os.remove(obj)
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force or bool(extra), verbose=True, extra_flags=extra))
