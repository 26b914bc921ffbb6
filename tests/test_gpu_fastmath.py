"""The FMA-pipe 2^x of the one-tile attention kernel (Cody-Waite reduction
to j + f with |f| <= 1/2 and a fitted cubic for 2^f) against exact values:
relative error at most 7.5e-5 wherever 2^x is above the smallest normal
fp32 number, non-negative and below 2^-125 elsewhere (inputs below -126 are
clamped there), through the C ABI's self-test entry point."""
import numpy as np
import pytest
import torch

import adaptive_vector_quantized_b200 as avq

pytestmark = pytest.mark.gpu


def test_exp2_poly_error_bound():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.uniform(-127.0, 0.0, 400000),      # the range the attention kernel feeds it
        rng.uniform(0.0, 24.0, 100000),        # children above the parents' maximum (before a rescale)
        np.arange(-126, 25, dtype=np.float64),  # integers: f = 0
        np.arange(-126, 24, dtype=np.float64) + 0.5,  # f at the ends of the reduction interval
        np.arange(-126, 24, dtype=np.float64) - 0.5,
        [0.0, -0.0, 1e-8, -1e-8, 0.25, -0.25],
    ]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    y = avq.avq_selftest_exp2(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    avq.avq_check_device()
    exact = np.exp2(x.astype(np.float64))
    normal = exact > 2.0 ** -126
    rel = np.abs(y[normal] - exact[normal]) / exact[normal]
    assert rel.max() <= 7.6e-5, rel.max()
    # below the normal range the result is tiny and never negative
    assert np.all(y[~normal] >= 0.0) and np.all(y[~normal] <= 2.0 ** -125)


def test_exp2_poly_clamps_low_inputs():
    x = torch.tensor([-126.0, -126.5, -127.0, -128.0, -200.0, -1e30], dtype=torch.float32, device="cuda")
    y = avq.avq_selftest_exp2(x).cpu().numpy()
    avq.avq_check_device()
    assert not np.isnan(y).any()
    assert np.all(y >= 0.0) and np.all(y <= 2.0 ** -125)


def test_exp2_selftest_rejects_odd_length():
    x = torch.zeros(3, dtype=torch.float32, device="cuda")
    with pytest.raises(avq.AVQError):
        avq.avq_selftest_exp2(x)
