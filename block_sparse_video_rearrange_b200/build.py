"""Builds librf.so (the CUDA path) in-tree with nvcc for sm_100a.

Usage: python -m block_sparse_video_rearrange_b200.build [-v]
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librf.so")
SOURCES = ["rf_plan.cu", "rf_rearrange.cu", "rf_select.cu", "rf_attn.cu", "rf_noalloc.cu", "rf_selftest.cu"]


def nvcc_path():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(ptxas_verbose=False, out=LIB, defines=()):
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
           "-shared", "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", out]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [f"-D{d}" for d in defines]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    return cmd


def build(verbose=False, force=False):
    """Compile librf.so unless it is newer than every source; returns its path."""
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "rf.h")]
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in deps):
        return LIB
    tmp = LIB + ".tmp"
    res = subprocess.run(command(verbose, tmp), capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building librf.so")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
