"""The FMA-pipe exp2 polynomial used in the prefill softmax, against the
exact value (fp64) and against CUDA's exp2f, on a dense grid of inputs."""

import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def probe(cuda_device):
    d = tempfile.mkdtemp(prefix="exp2probe_")
    so = os.path.join(d, "exp2_probe.so")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                    "--use_fast_math", "-Xcompiler", "-fPIC", "-shared", "-o", so,
                    os.path.join(HERE, "cuda", "exp2_probe.cu")], check=True)
    lib = ctypes.CDLL(so)
    lib.exp2_probe.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int]
    return lib


def run(probe, x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    yp, yk, yr = np.empty_like(x), np.empty_like(x), np.empty_like(x)
    assert probe.exp2_probe(x.ctypes.data, yp.ctypes.data, yk.ctypes.data, yr.ctypes.data, x.size) == 0
    return yp, yk, yr


def test_relative_error_bound(probe):
    # the softmax feeds x = s*scale*log2(e) - m <= 8
    x = np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float32)
    yp, yk, yr = run(probe, x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(yp - exact) / exact
    assert rel.max() <= 8e-5, rel.max()
    # the packed two-lane form used by the softmax gives the same values
    assert (np.abs(yk - exact) / exact).max() <= 8e-5
    # and it agrees with CUDA's exp2f to the same bound
    assert (np.abs(yp - yr.astype(np.float64)) / exact).max() <= 1e-4


def test_special_values(probe):
    x = np.array([-np.inf, -1000.0, -126.0, -125.5, 0.0, 1.0, -1.0, 8.0, 0.5, -0.5], dtype=np.float32)
    yp, yk, _ = run(probe, x)
    # packed form clamps: inputs below -125 give ~2^-125 instead of 0
    assert np.all(yk[:4] <= 2.0 ** -124) and np.all(yk[:4] >= 0.0)
    assert np.allclose(yk[4:], yp[4:], rtol=1e-6)
    assert yp[0] == 0.0 and yp[1] == 0.0 and yp[2] == 0.0 and yp[3] == 0.0
    assert abs(yp[4] - 1.0) <= 8e-5 and abs(yp[5] - 2.0) <= 2 * 8e-5 and abs(yp[7] - 256.0) <= 256 * 8e-5
    assert np.all(np.isfinite(yp))
