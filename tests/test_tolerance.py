"""CPU checks of the bf16 storage bound the GPU parity tests use (gpu_helpers.bf16_round_halfwidth).

The bound says a bf16-stored device value `got` is the rounding of some real within the stated
fraction of RMS of the oracle value: |got - ref| <= frac * RMS + the half-width of got's rounding
interval on the side facing ref.  These tests pin the half-width against torch's own float -> bf16
rounding: every real rounds to a value whose interval contains it, and the interval is no wider
than that (a real just outside it rounds to another value).
"""
import numpy as np
import torch

from gpu_helpers import bf16_round_halfwidth


def _bf16(x):
    """float32 -> bf16, one rounding (as the kernels store their float32 results); the inputs are
    made float32 first, so torch's conversion rounds once."""
    x32 = np.asarray(x, np.float32)
    return torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()


def test_halfwidth_contains_every_rounding():
    g = np.random.default_rng(3)
    r = np.concatenate([g.standard_normal(200000) * 10.0 ** g.integers(-6, 6, 200000),
                        np.ldexp(1.0, g.integers(-20, 20, 5000)) * (1 + g.uniform(-1e-3, 1e-3, 5000))])
    r = r.astype(np.float32).astype(np.float64)
    got = _bf16(r)
    assert np.all(np.abs(got - r) <= bf16_round_halfwidth(got, r))


def test_halfwidth_is_tight():
    g = np.random.default_rng(4)
    got = _bf16(g.standard_normal(20000) * 8.0)
    got = got[got != 0]
    for side in (-1.0, 1.0):
        ref = got + side * np.abs(got) * 1e-9          # which side of got the interval is measured on
        hw = bf16_round_halfwidth(got, ref)
        outside = got + side * hw * (1 + 1e-3)
        assert np.all(_bf16(outside) != got)
        inside = got + side * hw * (1 - 1e-3)
        assert np.all(_bf16(inside) == got)


def test_halfwidth_below_a_power_of_two():
    # 1.0 is a bf16 value; the next value below is 1 - 2**-8, so reals down to 1 - 2**-9 round to 1
    got = np.array([1.0, 1.0, 8.0])
    ref = np.array([0.99, 1.01, 7.9])
    np.testing.assert_array_equal(bf16_round_halfwidth(got, ref), [2.0 ** -9, 2.0 ** -8, 2.0 ** -6])
