"""Builds libvattn.so (sm_100a) in-tree with nvcc.

    python video_dit_local_b200/build.py [-v] [--debug]

Each .cu file under csrc/ is compiled to an object in parallel, then linked
into video_dit_local_b200/libvattn.so (cudart linked statically, no libcuda
link dependency: the TMA encoder is fetched from the driver at run time).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libvattn.so")
# Debug build: the same library compiled with -DVATTN_DEBUG=1 (device-side
# bounds checks on every computed row, tile and TMA coordinate; a failed check
# reports VATTN_ERR_DEVICE_BOUNDS through vattn_get_status).  The binding
# loads it instead of LIB when VATTN_DEBUG_BUILD=1 is set in the environment.
LIB_DEBUG = os.path.join(HERE, "libvattn_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC,-O2",
    "-Xptxas", "-v",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _up_to_date(srcs, lib=LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "vattn.h")]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    srcs = _sources()
    lib = LIB_DEBUG if debug else LIB
    if not force and _up_to_date(srcs, lib):
        return lib
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    if debug:
        extra_flags = (*extra_flags, "-DVATTN_DEBUG=1")

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(compile_one, srcs))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    objs = [o for o, _ in results]
    tmp = lib + ".tmp"
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs],
                       capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
