"""The bf16 acceptance bar's allowance for the output's own rounding.

The bar bounds |got - ref| less half an ulp of the bf16 output (the most that
rounding the exact value to bf16 moves it). Pinned against torch's bf16
rounding: every rounded value is within that half ulp of its source, and the
half ulp is half the gap to the next bf16 value.
"""
import numpy as np
import pytest
import torch

from tests import gpu_helpers as G


def test_half_ulp_is_half_the_bf16_spacing():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 300, 2000), rng.uniform(-1e-3, 1e-3, 2000),
                        [1.0, 2.0, 4.0, 4.21875, -4.20794, 7.99, 8.0, 1e-30]])
    b = torch.tensor(x, dtype=torch.float64).to(torch.bfloat16)
    up = torch.nextafter(b.abs(), torch.full_like(b, float("inf")))
    spacing = (up.double() - b.abs().double()).numpy()
    half = G.bf16_half_ulp(b.double().numpy())
    nz = b.double().numpy() != 0
    assert np.allclose(half[nz], spacing[nz] / 2, rtol=0, atol=0)
    # rounding moves a value by at most that half ulp of the result
    assert np.all(np.abs(b.double().numpy() - x) <= half)


def test_correctly_rounded_output_passes_and_one_ulp_off_fails():
    ref = np.concatenate([[-4.20794], np.random.default_rng(4).normal(0, 0.05, 4000)])
    got = torch.tensor(ref, dtype=torch.float64).to(torch.bfloat16).double().numpy()
    assert abs(got[0] - ref[0]) > G.BF16_MAX_ABS  # the rounding alone exceeds 1e-2 here
    G.check_tolerance(got, ref, "bf16")
    bad = got.copy()
    bad[0] = -4.21875 - 2 * 0.015625 * 2  # two ulps away: 0.07 of arithmetic error
    with pytest.raises(AssertionError):
        G.check_tolerance(bad, ref, "bf16")
