"""The prefill kernel's FMA-pipe exponential (Cody-Waite reduction + degree-4
minimax polynomial) against exact 2^x and against the MUFU ex2.approx it
shares the work with."""
import numpy as np
import pytest
import torch

from polar_attention_b200 import native

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound(cuda_ok):
    x = np.concatenate([np.linspace(-125.9, 8.0, 2_000_000), np.arange(-125, 9, 0.5),
                        np.linspace(-1, 1, 100001)]).astype(np.float32)
    x = x[: x.size // 2 * 2]
    poly, mufu = native.selftest_exp2(torch.from_numpy(x).cuda())
    exact = np.exp2(x.astype(np.float64))
    rp = np.abs(poly.cpu().numpy().astype(np.float64) / exact - 1.0)
    rm = np.abs(mufu.cpu().numpy().astype(np.float64) / exact - 1.0)
    assert rp.max() < 5e-6, f"polynomial relative error {rp.max():.3e}"
    # the two agree to within both error bounds
    assert np.max(np.abs(poly.cpu().numpy() / mufu.cpu().numpy() - 1.0)) < 6e-6
    assert rm.max() < 1e-6
