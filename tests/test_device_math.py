"""The prefill softmax computes part of its exponentials with the library's own polynomial on the FMA pipe
(range reduction by rounding to nearest, a degree-3 fit of 2^f on [-1/2, 1/2]) and the rest with the
special-function unit's ex2.  pa_selftest_exp2 evaluates both on the GPU; here both are held to error bounds
against fp64 exp2 on a dense grid of the inputs the softmax produces (x <= 8 after the lazy maximum, far
below zero for keys that barely count, -inf for masked keys)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_325_b200 as pa

pytestmark = pytest.mark.gpu


def test_polynomial_exp2_within_its_bound(cuda_lib):
    x = np.concatenate([np.linspace(-125.0, 9.0, 1_000_001), np.random.default_rng(3).uniform(-30, 9, 100_000)])
    xt = torch.tensor(x, dtype=torch.float32, device="cuda:0")
    y_poly, y_sfu = pa.pa_selftest_exp2(xt)
    torch.cuda.synchronize()
    xf = xt.double().cpu().numpy()
    ref = np.exp2(xf)
    rel_poly = np.abs(y_poly.double().cpu().numpy() - ref) / ref
    rel_sfu = np.abs(y_sfu.double().cpu().numpy() - ref) / ref
    # far below the 2^-9 relative spacing of the bf16 values P is rounded to
    assert rel_poly.max() < 1e-4, rel_poly.max()
    assert rel_sfu.max() < 1e-4, rel_sfu.max()


def test_polynomial_exp2_of_masked_and_tiny_inputs(cuda_lib):
    x = torch.tensor([-float("inf"), -1e30, -200.0, -126.0, -125.0, -124.5], dtype=torch.float32, device="cuda:0")
    y_poly, y_sfu = pa.pa_selftest_exp2(x)
    torch.cuda.synchronize()
    yp = y_poly.double().cpu().numpy()
    # clamped to 2^-125 (a normal float): no sum in fp32 can tell it from 0, and it is never NaN or negative
    assert np.all(np.isfinite(yp)) and np.all(yp >= 0) and np.all(yp <= 2.0 ** -124)
    assert y_sfu[0].item() == 0.0
