"""The FMA-pipe exponential of the FP8 forward pass (one pair of probabilities
in four is computed as 2^n * p(f), x = n + f, p a cubic fitted for least
maximum relative error on |f| <= 1/2) against 2^x in fp64.

Claimed: relative error at most 7.5e-5 on [-125, 0] (the arguments the
softmax produces: scaled score minus a running max), plus the fp32 rounding of
the evaluation; exactly 0 below -125 (masked keys, whose argument is -inf).
"""
import numpy as np
import pytest
import torch

import exact_attention_157_b200 as ea

pytestmark = pytest.mark.gpu

REL = 7.5e-5 + 4 * 2.0 ** -24  # the fit's error plus a few fp32 roundings


def run(x):
    y = ea.exp2_poly(torch.from_numpy(x).to("cuda:0"))
    ea.check_device_status()
    return y.cpu().numpy()


def test_relative_error_over_the_softmax_range():
    # dense grid over [-125, 0] plus the points where f = +-1/2 and the integers
    x = np.concatenate([np.linspace(-125.0, 0.0, 1 << 22, dtype=np.float32),
                        np.arange(-125, 1, dtype=np.float32),
                        np.arange(-124.5, 0.0, 1.0, dtype=np.float32),
                        np.nextafter(np.arange(-124.5, 0.0, 1.0, dtype=np.float32), np.float32(0.0))])
    y = run(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    worst = int(np.argmax(rel))
    print(f"exp2_poly max relative error {rel.max():.3e} at x = {x[worst]}")
    assert rel.max() <= REL, f"relative error {rel.max()} at x = {x[worst]}"
    # a cubic that matched only at the nodes would show here: the error is not tiny everywhere
    assert rel.max() > 1e-6


def test_slightly_positive_arguments():
    """The lazy rescale lets arguments reach +2 (FP8 threshold) above the stale max,
    plus the 2^6 P shift: up to about +8."""
    x = np.linspace(0.0, 8.0, 1 << 16, dtype=np.float32)
    y = run(x)
    assert (np.abs(y / np.exp2(x.astype(np.float64)) - 1.0) <= REL).all()


def test_below_minus_125_is_zero():
    x = np.array([-np.inf, -1e30, -1000.0, -126.0, -125.5, np.nextafter(np.float32(-125.0), np.float32(-200.0))],
                 dtype=np.float32)
    assert (run(x) == 0.0).all()
    # -125 itself stays normal
    y = run(np.array([-125.0], dtype=np.float32))[0]
    assert abs(y / 2.0 ** -125 - 1.0) <= REL


def test_odd_count_and_empty():
    x = np.array([-1.0, -2.0, -3.0], dtype=np.float32)
    np.testing.assert_allclose(run(x), [0.5, 0.25, 0.125], rtol=REL)
    assert run(np.zeros(0, dtype=np.float32)).size == 0
