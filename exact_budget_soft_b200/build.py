"""Build the CUDA library liblapsum.so in-tree (sm_100a) with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblapsum.so")
# the checked build: device bounds tests on computed indices and guard words
# around the workspace (-DLAPSUM_CHECKED), loaded when LAPSUM_CHECKED=1
LIB_CHECKED = os.path.join(HERE, "liblapsum_checked.so")
SOURCES = ["lapsum_api.cu", "k_rows.cu", "k_bracket.cu", "k_radix.cu", "k_band.cu", "k_noalloc.cu", "k_shard.cu"]
HEADERS = ["lapsum_internal.h", "lapsum_kernels.h", "lapsum_device.cuh", "scan_solve.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(HERE, "..", "include", "lapsum.h"))
    deps.append(__file__)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not (force or _stale(lib)):
        return lib
    objs = []
    bdir = os.path.join(HERE, "_build_checked" if checked else "_build")
    os.makedirs(bdir, exist_ok=True)
    procs = []
    for src in SOURCES:
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, *(["-DLAPSUM_CHECKED"] if checked else []), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
        objs.append(obj)
    failed = False
    for src, p in procs:
        out, _ = p.communicate()
        text = out.decode()
        if text.strip() and (verbose or p.returncode):
            sys.stderr.write(f"--- {src}\n{text}")
        if p.returncode:
            failed = True
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC", "-o", tmp, *objs])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
