"""Accuracy of the device exponentials and activations against float64
(needs a GPU).

The paired polynomial 2^x (FMA pipe) and ex2.approx (special-function
unit) both feed the decay exp(Delta A); each must stay within a few fp32
ulps of 2^x over the range the scan uses, give exactly 1 at x = 0 (padded
steps are identities) and flush to ~0 below 2^-126.  The step size
softplus(x) = max(x, 0) + log1p(e^-|x|) and the gate silu(z) must hold a
relative error of about 1e-6 (plus the rounding of the exponent, which
grows with |x|), far inside the 1e-4 parity bound on y.
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
    lib.eval_activations.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int]
    lib.eval_activations.restype = ctypes.c_int

    def run(x):
        x = torch.as_tensor(np.asarray(x, dtype=np.float32), device="cuda")
        n = x.numel() - x.numel() % 2
        poly = torch.empty_like(x)
        mufu = torch.empty_like(x)
        assert lib.eval_exp2(x.data_ptr(), poly.data_ptr(), mufu.data_ptr(), n) == 0
        torch.cuda.synchronize()
        return poly[:n].cpu().numpy(), mufu[:n].cpu().numpy()

    def act(x):
        x = torch.as_tensor(np.asarray(x, dtype=np.float32), device="cuda")
        n = x.numel() - x.numel() % 2
        outs = [torch.empty_like(x) for _ in range(4)]
        assert lib.eval_activations(x.data_ptr(), *[o.data_ptr() for o in outs], n) == 0
        torch.cuda.synchronize()
        return [o[:n].cpu().numpy() for o in outs]
    run.act = act
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


def _softplus64(x):
    x = x.astype(np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def test_softplus_relative_error(evaluator):
    rng = np.random.default_rng(1)
    x = np.concatenate([np.linspace(-87.0, 87.0, 400002),
                        rng.normal(-4.0, 2.0, 200000),
                        [0.0, -0.0, 1e-30, -1e-30]]).astype(np.float32)
    sp_pair, sp_scalar, _, _ = evaluator.act(x)
    xs = x[:len(sp_pair)]
    ref = _softplus64(xs)
    bound = 1e-6 + 8e-8 * np.abs(xs.astype(np.float64))
    for got in (sp_pair, sp_scalar):
        rel = np.abs(got / ref - 1)
        assert np.all(rel <= bound), float(np.max(rel / bound))


def test_softplus_limits(evaluator):
    x = np.array([np.inf, -np.inf, 100.0, -100.0, np.nan, 0.0], dtype=np.float32)
    sp_pair, sp_scalar, _, _ = evaluator.act(x)
    for got in (sp_pair, sp_scalar):
        assert got[0] == np.inf and got[1] == 0.0 and got[2] == 100.0
        assert 0.0 <= got[3] < 1e-37
        assert np.isnan(got[4])
        assert abs(got[5] / np.log(2.0) - 1) < 1e-6


def test_silu_relative_error(evaluator):
    z = np.linspace(-80.0, 80.0, 400002).astype(np.float32)
    _, _, si_pair, si_scalar = evaluator.act(z)
    zs = z[:len(si_pair)].astype(np.float64)
    ref = zs / (1.0 + np.exp(-zs))
    bound = 2e-6 + 8e-8 * np.abs(zs)
    nz = ref != 0
    for got in (si_pair, si_scalar):
        rel = np.abs(got[nz] / ref[nz] - 1)
        assert np.all(rel <= bound[nz]), float(np.max(rel / bound[nz]))
