"""The C ABI from plain C: tests/c/abi_example.c includes only ccv3d.h and
the CUDA runtime header and links libccv3d.so -- no Python, no torch on its
path.  Without a GPU it checks the host planner; with one (the gpu test) it
runs a forward on zero inputs and checks out == bias and new_cache == 0."""
import os
import shutil
import subprocess

import pytest

from causal_conv3d_video_b200 import ccv3d

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA = "/usr/local/cuda"


def _build(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(ccv3d.LIB_PATH)
    exe = str(tmp_path / "abi_example")
    subprocess.check_call([cc, "-std=c99", "-O1", "-Wall", "-Werror",
                           os.path.join(HERE, "c", "abi_example.c"),
                           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                           "-L", libdir, "-lccv3d", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                           "-Wl,-rpath," + libdir, "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
                           "-o", exe])
    return exe


def test_c_program_plans_without_python(tmp_path):
    import torch
    if torch.cuda.is_available():
        pytest.skip("the GPU variant runs the forward")
    exe = _build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "kernel=tc_pair T_o=1 H_o=90 W_o=160" in r.stdout
    assert "host-only checks passed" in r.stdout


@pytest.mark.gpu
def test_c_program_runs_forward(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "forward ok: mismatches=0 calls=1 tc=1" in r.stdout
