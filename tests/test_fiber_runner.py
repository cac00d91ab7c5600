"""The host fiber runner that executes CUDA-style kernel bodies in the *_host
tests: a warp butterfly gives the warp's sum in every lane, and a barrier that
not every thread reaches stops the process instead of passing silently."""
import ctypes
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def so(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ is not available")
    out = str(tmp_path_factory.mktemp("runner") / "runner_selftest.so")
    subprocess.run([gxx, "-O1", "-std=c++17", "-fPIC", "-shared", "-o", out,
                    os.path.join(HERE, "cuda_host", "runner_selftest.cpp")], check=True)
    return out


def test_butterfly_sums_each_warp(so):
    lib = ctypes.CDLL(so)
    n = 128
    out = np.zeros(n, np.float32)
    assert lib.runner_butterfly(n, out.ctypes.data_as(ctypes.c_void_p)) == 0
    warp_sum = lambda w: sum(range(32 * w + 1, 32 * w + 33))
    expect = np.array([warp_sum(((t + 32) % n) // 32) for t in range(n)], np.float32)
    assert np.array_equal(out, expect)


def test_divergent_barrier_aborts(so):
    code = f"import ctypes; ctypes.CDLL({so!r}).runner_divergent_barrier()"
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=60)
    assert r.returncode != 0 and "barrier divergence" in r.stderr
