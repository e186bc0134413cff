"""Builds libmlstm.so in-tree with nvcc for sm_100a (B200), and libmlstm_checked.so: the same
library with the bounds checks of the tensor-core prefill compiled in (MLSTM_BOUNDS_CHECK)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmlstm.so")
LIB_CHECKED = os.path.join(PKG, "libmlstm_checked.so")
# sources whose objects differ in the bounds-checked build (the others are linked as they are)
CHECKED_SOURCES = ("chunkwise_tc.cu", "gdn2_tc.cu", "mlstm_api.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(LIB_CHECKED):
        return True
    t = min(os.path.getmtime(LIB), os.path.getmtime(LIB_CHECKED))
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every csrc/*.cu (in parallel, objects under _build/) and link them into
    linear_recurrent_token_b200/libmlstm.so (static cudart); compile CHECKED_SOURCES again with
    -DMLSTM_BOUNDS_CHECK and link libmlstm_checked.so from those and the other objects."""
    if not force and not _stale():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    objdir = os.path.join(ROOT, "_build")
    os.makedirs(os.path.join(objdir, "checked"), exist_ok=True)
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]

    def compile_one(job):
        src, checked = job
        obj = os.path.join(objdir, "checked" if checked else "", os.path.basename(src) + ".o")
        cmd = [nvcc()] + compile_flags + (["-DMLSTM_BOUNDS_CHECK"] if checked else []) \
            + ["-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        return obj

    srcs = sources()
    jobs = [(s, False) for s in srcs] + [(s, True) for s in srcs if os.path.basename(s) in CHECKED_SOURCES]
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(compile_one, jobs))
    plain = objs[:len(srcs)]
    checked = {os.path.basename(o)[:-2]: o for o in objs[len(srcs):]}
    variants = ((LIB, plain), (LIB_CHECKED, [checked.get(os.path.basename(o)[:-2], o) for o in plain]))
    for lib, lib_objs in variants:
        tmp = lib + ".tmp%d" % os.getpid()
        cmd = [nvcc()] + NVCC_FLAGS + ["-o", tmp] + lib_objs
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
