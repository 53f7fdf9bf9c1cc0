"""Pins of the parity helpers in tests/parity.py (CPU)."""

import numpy as np
import torch

from parity import bf16_band, bf16_rne, check_fwd, fwd_figures


def test_bf16_rne_matches_torch_rounding_of_fp32_values():
    # torch rounds float32 -> bfloat16 to nearest even; on values that are exact
    # in float32 the helper must agree bit for bit, ties and binade edges included
    g = torch.Generator().manual_seed(0)
    x = torch.cat([torch.randn(200000, generator=g) * 4.0,
                   torch.tensor([1.0 + 2**-8, 1.0 + 3 * 2**-8, -(1.0 + 2**-8), 255.5 / 128, 2.0 - 2**-9,
                                 3 * 2**-130, 0.0, -0.0, 6.5e4, 2**-126])])
    want = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = bf16_rne(x.to(torch.float64).numpy())
    assert np.array_equal(got, want)


def test_band_is_the_rounding_of_every_value_within_tolerance():
    # brute force: the band's ends are the smallest and largest bf16 roundings
    # of points within 1e-2 of the reference
    rng = np.random.default_rng(1)
    ref = rng.normal(size=300) * 3
    lo, hi = bf16_band(ref)
    pts = ref[:, None] + np.linspace(-1e-2, 1e-2, 2001)[None, :]
    r = bf16_rne(pts)
    assert np.array_equal(lo, r.min(axis=1)) and np.array_equal(hi, r.max(axis=1))


def test_band_check_admits_rounded_results_and_rejects_larger_errors():
    rng = np.random.default_rng(2)
    ref = rng.normal(size=(1, 1, 64, 16)) * 3
    lse = np.zeros((1, 1, 64))
    ok = bf16_rne(ref + rng.uniform(-9.9e-3, 9.9e-3, size=ref.shape))
    assert fwd_figures(ok, lse, ref, lse)["o_outside_band"] == 0
    check_fwd(ok, lse, ref, lse, "within")
    bad = ok.copy()
    bad[0, 0, 5, 3] = bf16_rne(ref[0, 0, 5, 3] + 0.03)
    assert fwd_figures(bad, lse, ref, lse)["o_outside_band"] == 1
