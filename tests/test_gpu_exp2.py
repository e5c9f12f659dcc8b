"""The library's FMA-pipe exponential, which the attention kernels can use
for a share of their softmax weights (they currently take all of them from
MUFU, which measured faster), checked on the device against its stated
error bound (relative error <= 7.5e-5 against exact 2^x, from the minimax
fit of the polynomial) and against the MUFU exponential it would stand in
for."""
import ctypes as C

import numpy as np
import pytest
import torch

from dynamic_block_sparse_stats_b200 import _lib

pytestmark = pytest.mark.gpu


def _eval(x):
    lib = _lib.load()
    xd = torch.as_tensor(x, dtype=torch.float32, device="cuda")
    yp, ym = torch.empty_like(xd), torch.empty_like(xd)
    _lib.check(lib.prism_diag_exp2(C.c_void_p(xd.data_ptr()), C.c_void_p(yp.data_ptr()), C.c_void_p(ym.data_ptr()),
                                   xd.numel(), torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return yp.cpu().numpy().astype(np.float64), ym.cpu().numpy().astype(np.float64)


def test_poly_exp2_error_bound_over_the_softmax_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 64.0, 400_001), rng.uniform(-30, 10, 200_001),
                        np.arange(-125, 65, dtype=np.float64),                   # integers: f = 0
                        np.arange(-125, 64) + 1 - 2.0 ** -17]).astype(np.float32)  # just below integers
    yp, ym = _eval(x)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(yp / exact - 1.0)
    assert rel.max() <= 7.6e-5, rel.max()
    # against the MUFU result, which is within ~2^-22 of exact
    assert np.abs(yp / ym - 1.0).max() <= 7.7e-5


def test_poly_exp2_clamps_like_the_values_it_replaces():
    x = np.array([-1e30, -1000.0, -126.0, -125.5, 64.5, 200.0, 1e30], dtype=np.float32)
    yp, _ = _eval(x)
    # below the clamp the result is below 2^-124 (zero in fp16); above it is 2^64 (inf in fp16)
    assert (yp[:4] >= 0).all() and (yp[:4] < 2.0 ** -124).all()
    assert np.allclose(yp[4:], 2.0 ** 64, rtol=1e-4)
    assert np.isinf(np.float16(yp[4:])).all() and (np.float16(yp[:4]) == 0).all()


def test_poly_exp2_odd_length():
    x = np.array([0.5, -2.25, 3.0], dtype=np.float32)
    yp, ym = _eval(x)
    np.testing.assert_allclose(yp, np.exp2(x.astype(np.float64)), rtol=7.6e-5)
