"""Build libflint_moe.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
SO = os.path.join(PKG, "libflint_moe.so")
OBJ_DIR = os.path.join(PKG, "_build")
# translation units, compiled in parallel and linked into one shared library
SOURCES = ["flint_moe.cu", "tok1.cu", "tokn.cu", "lmhead.cu", "attn.cu", "attn_decode.cu", "ep.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return files


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(SO):
        so_time = os.path.getmtime(SO)
        if all(os.path.getmtime(f) <= so_time for f in _inputs()):
            return SO
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ_DIR, exist_ok=True)
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(OBJ_DIR, os.path.splitext(src)[0] + f".{os.getpid()}.o")
        cmd = [nvcc, *NVCC_FLAGS, f"-I{INCLUDE}", "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        objs.append(obj)
        procs.append(subprocess.Popen(cmd))
    failed = [p.wait() for p in procs]
    if any(failed):
        for o in objs:
            if os.path.exists(o):
                os.unlink(o)
        raise subprocess.CalledProcessError(max(failed), "nvcc")
    tmp = SO + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, "-shared", *objs, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    for o in objs:
        os.unlink(o)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
