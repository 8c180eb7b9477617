"""Build libccv3d.so in-tree with nvcc for sm_100a (B200).

    python -m causal_conv3d_video_b200.build [--force] [--verbose-ptxas]

The library is a single translation unit (csrc/ccv3d.cu) exporting the C ABI
declared in include/ccv3d.h.  The CUDA runtime is linked statically; the
driver's cuTensorMapEncodeTiled is reached through cudaGetDriverEntryPoint,
so no -lcuda is needed at link time.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libccv3d.so")
# the bounds-checked build (-DCCV3D_CHECKED): every computed global address is
# range-checked before use; a violation is reported as CCV3D_ERR_BOUNDS
CHECKED_LIB_PATH = os.path.join(LIB_DIR, "libccv3d_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libccv3d")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*"))) + [
        os.path.join(ROOT, "include", "ccv3d.h")]


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    path = CHECKED_LIB_PATH if checked else LIB_PATH
    if not force and up_to_date(path):
        return path
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"),
           os.path.join(CSRC, "ccv3d.cu"), "-o", tmp]
    if checked:
        cmd[1:1] = ["-DCCV3D_CHECKED"]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--checked", action="store_true", help="build libccv3d_checked.so")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, checked=a.checked))
    sys.exit(0)
