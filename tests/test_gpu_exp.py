"""The float64 exponential of the mask cut (csrc/exp_nonpos.cuh, Cody-Waite
reduction and a degree-13 Taylor polynomial) against CUDA's exp on the GPU:
within two units in the last place of it everywhere on [-30, 0] (each is
within about one of e^x), and the integer
masses floor(e^x * 2^40) it yields equal to those from CUDA's exp on all but
a vanishing share of arguments (a difference needs e^x * 2^40 within an ulp
of an integer).  A test-only kernel is compiled from tests/exp_check.cu."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def lib():
    out = os.path.join(tempfile.mkdtemp(), "libexp_check.so")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-o", out,
                           os.path.join(HERE, "exp_check.cu")])
    L = ctypes.CDLL(out)
    L.exp_check.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    return L


def _ulp(v):
    return np.ldexp(1.0, np.frexp(v)[1] - 53)


def test_exp_nonpos_matches_cuda_exp(lib):
    rng = np.random.default_rng(0)
    x = np.concatenate([-np.sort(rng.random(1 << 20)) * 30.0, -rng.random(1 << 18) * 1e-3,
                        np.array([0.0, -0.5 * np.log(2), -np.log(2), -27.72588722239781,
                                  -28.0, -30.0, -np.inf])])
    xd = torch.from_numpy(x).cuda()
    mine, ref = torch.empty_like(xd), torch.empty_like(xd)
    assert lib.exp_check(xd.data_ptr(), mine.data_ptr(), ref.data_ptr(), x.size) == 0
    torch.cuda.synchronize()
    m, c = mine.cpu().numpy(), ref.cpu().numpy()
    fin = np.isfinite(x)
    err = np.abs(m[fin] - c[fin]) / _ulp(c[fin])
    assert err.max() <= 2.0, err.max()  # each within about one ulp of e^x
    # the masses the cut uses
    um = np.floor(m[fin] * 2.0 ** 40)
    uc = np.floor(c[fin] * 2.0 ** 40)
    assert np.mean(um != uc) < 1e-4
    assert np.all(np.abs(um - uc) <= 1)
    assert m[x == 0.0][0] == 1.0
    assert np.floor(m[-1] * 2.0 ** 40) == 0.0  # -inf: no mass
