"""Build the CUDA library in-tree: selective_scan_ss2d_b200/_lib/libss2d_b200.so.

nvcc compiles for sm_100a only (B200); the CUDA runtime is linked
statically so the library does not depend on which libcudart the host
process has loaded.  ``python -m selective_scan_ss2d_b200.build`` rebuilds.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIBDIR, "libss2d_b200.so")
SOURCES = ["ss2d_capi.cu", "ss2d_launch.cu", "ss2d_noalloc.cu", "ss2d_scan_bf16.cu",
           "ss2d_scan_f32.cu", "ss2d_scan_f16.cu", "ss2d_backward.cu", "ss2d_front.cu"]
HEADERS = ["ss2d_kernels.cuh", "ss2d_scan.cuh", "ss2d_front.cuh", "ss2d_scan_launch.cuh", "ss2d_launch.h",
           "ss2d_params.h", "ss2d_backward.cuh", "ss2d_bwd_params.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs() -> list[str]:
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "ss2d.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(LIBDIR, exist_ok=True)
    # every translation unit compiles in its own nvcc process, all at once
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(LIBDIR, os.path.splitext(src)[0] + f".{os.getpid()}.o")
        cmd = [nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
               "-Xptxas", "-v", "-I", INCLUDE, "-I", CSRC, "-c", os.path.join(CSRC, src),
               "-o", obj]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                            text=True)))
        objs.append(obj)
    log_lines, failed = [], []
    for src, pr in procs:
        out, _ = pr.communicate()
        log_lines.append(out)
        if pr.returncode != 0:
            failed.append(src)
            sys.stderr.write(out)
    if failed:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
        raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc link failed")
    os.replace(tmp, LIB)
    with open(os.path.join(LIBDIR, "ptxas.log"), "w") as f:
        f.write("\n".join(log_lines))
    for o in objs:
        os.remove(o)
    if verbose:
        print("\n".join(log_lines))
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
