"""Bounds on the GEMM epilogues' own approximations, evaluated on the GPU by
the library's self-test kernel beside CUDA's functions:

  tanh_fast(x) = 1 - 2 / (2^(2 x log2 e) + 1)   (the softcap c tanh(z / c))
  ex2a(x)      = the ex2.approx.ftz instruction (every exponential)

tanh_fast has an absolute error of a few fp32 ulps of 1 (the subtraction
from 1 loses relative accuracy near 0, never absolute), so the softcap's
y = c tanh(z/c) is off by at most c times that.  ex2a's relative error stays
within a few 2^-23 for outputs above the fp32 normal range's floor and it
flushes what lies below to 0."""
import numpy as np
import pytest
import torch

from linear_cross_entropy_tiles_b200 import binding

pytestmark = pytest.mark.gpu


def test_tanh_fast_absolute_error(cuda_device):
    x = torch.cat([torch.linspace(-20, 20, 400001), torch.logspace(-8, 1.5, 20001),
                   -torch.logspace(-8, 1.5, 20001),
                   torch.tensor([0.0, 1e-30, -1e-30, 88.0, -88.0, 1e4, -1e4])])
    r = binding.flce_selftest_approx(x.to(cuda_device)).cpu().double().numpy()
    ref = np.tanh(x.double().numpy())
    err_fast = np.abs(r[:, 0] - ref)
    err_lib = np.abs(r[:, 1] - ref)
    assert err_fast.max() <= 4e-7, err_fast.max()              # ~3 ulp of 1.0
    assert err_lib.max() <= 2e-7
    assert np.all(np.abs(r[:, 0]) <= 1.0)                      # saturates, never exceeds 1
    assert r[-2, 0] == 1.0 and r[-1, 0] == -1.0
    # the softcap at c = 30 (Gemma2): y is within 30 * 4e-7 of c tanh(z/c)
    assert (30 * err_fast).max() <= 1.2e-5


def test_ex2_approx_relative_error(cuda_device):
    x = torch.cat([torch.linspace(-126, 0, 500001), torch.linspace(0, 60, 60001),
                   torch.tensor([-150.0, -127.5, float("-inf")])])
    r = binding.flce_selftest_approx(x.to(cuda_device)).cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    normal = ref >= 2.0 ** -126
    rel = np.abs(r[normal, 2] - ref[normal]) / ref[normal]
    assert rel.max() <= 2.0 ** -21, rel.max()
    rel_lib = np.abs(r[normal, 3] - ref[normal]) / ref[normal]
    assert rel_lib.max() <= 2.0 ** -22
    assert np.all(r[~normal, 2] == 0.0)                        # flushed below the floor
    assert r[-1, 2] == 0.0                                     # 2^-inf = 0
