"""Accuracy of the device exponentials against float64 (needs a GPU).

The paired polynomial 2^x (FMA pipe) and ex2.approx (special-function
unit) both feed the decay exp(Delta A); each must stay within a few fp32
ulps of 2^x over the range the scan uses, give exactly 1 at x = 0 (padded
steps are identities) and flush to ~0 below 2^-126.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

from selective_state_space_48_b200 import builder

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def evaluator():
    tmp = tempfile.mkdtemp()
    so = os.path.join(tmp, "exp2_check.so")
    subprocess.run([builder.nvcc(), *builder.ARCH_FLAGS, "-O3", "-std=c++17",
                    "-Xcompiler", "-fPIC", "-shared", "-I", builder.CSRC,
                    os.path.join(HERE, "kernels", "exp2_check.cu"), "-o", so],
                   check=True, capture_output=True)
    lib = ctypes.CDLL(so)
    lib.eval_exp2.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    lib.eval_exp2.restype = ctypes.c_int

    def run(x):
        x = torch.as_tensor(np.asarray(x, dtype=np.float32), device="cuda")
        n = x.numel() - x.numel() % 2
        poly = torch.empty_like(x)
        mufu = torch.empty_like(x)
        assert lib.eval_exp2(x.data_ptr(), poly.data_ptr(), mufu.data_ptr(), n) == 0
        torch.cuda.synchronize()
        return poly[:n].cpu().numpy(), mufu[:n].cpu().numpy()
    return run


def test_relative_error_over_the_normal_range(evaluator):
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 127.0, 400002),
                        rng.uniform(-30, 0, 200000)]).astype(np.float32)
    poly, mufu = evaluator(x)
    ref = np.exp2(x[:len(poly)].astype(np.float64))
    assert np.max(np.abs(poly / ref - 1)) < 3e-7
    assert np.max(np.abs(mufu / ref - 1)) < 5e-7


def test_exact_points_and_underflow(evaluator):
    x = np.array([0.0, 0.0, 1.0, -1.0, 10.0, -20.0, -130.0, -1e6], dtype=np.float32)
    poly, mufu = evaluator(x)
    assert poly[0] == 1.0 and mufu[0] == 1.0
    assert poly[2] == 2.0 and poly[3] == 0.5 and poly[4] == 1024.0
    assert poly[5] == np.float32(2.0 ** -20)
    assert 0.0 <= poly[6] < 2.0 ** -125 and 0.0 <= poly[7] < 2.0 ** -125
