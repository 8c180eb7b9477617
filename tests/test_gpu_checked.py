"""The bounds-checked build (libccv3d_checked.so, compiled with -DCCV3D_CHECKED).

Every device address range a kernel computes -- generic loads and stores, the
persistent kernel's fp32 partial tiles and flags, bulk copies, the frame
coordinate of every TMA load and store -- is checked against the buffer it
indexes before use; a violation records CCV3D_ERR_BOUNDS in the call's status
and skips the access.  With no memory checker available, this build is how the
kernels' indexing is checked: the small-signature parity suite (every kernel
form, ragged tiles, strides, dilations, crop, batch 2, split stream-K tiles)
and the ring-buffer suite run against it in a child process, and each of
their tests already asserts that the call's status is CCV3D_OK.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _child(code_or_args, checked=True, timeout=1800):
    env = dict(os.environ)
    env.pop("CCV3D_TEST_OVERRIDES", None)
    if checked:
        env["CCV3D_LIBRARY"] = "checked"
    else:
        env.pop("CCV3D_LIBRARY", None)
    return subprocess.run([sys.executable] + code_or_args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_checked_build_records_violations():
    """The self-test hands the device checks an out-of-range byte range and
    index (never dereferenced): the checked build reports CCV3D_ERR_BOUNDS,
    the normal build, whose checks compile away, CCV3D_OK."""
    code = ("from causal_conv3d_video_b200 import ccv3d; import os; "
            "print(os.path.basename(ccv3d.LIB_PATH), ccv3d.ccv3d_selftest_bounds())")
    r = _child(["-c", code], checked=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["libccv3d_checked.so", "9"], r.stdout
    r = _child(["-c", code], checked=False)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["libccv3d.so", "0"], r.stdout


def test_small_parity_and_ring_suites_under_checked_build():
    r = _child(["-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                "tests/test_gpu_parity.py", "tests/test_gpu_ring.py", "tests/test_gpu_graph.py",
                "-k", "small or config1 or repeat or other_stream or refusals or ring_chunks "
                      "or graph"])
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail
