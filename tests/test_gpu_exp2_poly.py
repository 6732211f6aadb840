"""The FMA-pipe 2^x used for a share of the tensor-core attention's softmax exponentials
(spatten_selftest_exp2_poly), against float64 2^x.

Method (Cody-Waite reduction x = j + f, f in [-1/2, 1/2], degree-5 minimax polynomial of 2^f,
2^j by an exponent-field add): its float32 coefficients give 1.14e-7 relative error in exact
arithmetic and about 1.8e-7 with the roundings of the float32 Horner steps; the bound held here is
2^-22 (2.4e-7), the order of the ex2.approx instruction it stands in for.  Pins: a dense grid of
the softmax range [-126, 0], every float32 in [-1, 0] with a stride, integers (exact powers of two),
the clamp below -126, and the comparison with the ex2 path (torch.exp2 on the device).
"""
import numpy as np
import pytest
import torch

from gpu_helpers import lib

pytestmark = pytest.mark.gpu


def _run(S, x):
    xd = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    yd = torch.empty_like(xd)
    S.selftest_exp2_poly(xd, yd, xd.numel())
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def test_exp2_poly_relative_error_over_the_softmax_range(cuda):
    S = lib()
    g = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-126.0, 0.0, 1 << 22, dtype=np.float32),
                        (-g.random(1 << 20) * 126.0).astype(np.float32),
                        np.arange(-1.0, 0.0, 2.0 ** -20, dtype=np.float32),
                        np.float32([0.0, -0.5, -0.49999997, -0.50000006, -1.5, -125.5, -125.50001])])
    y = _run(S, x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= 2.0 ** -22, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"


def test_exp2_poly_exact_at_integers_and_clamped_below(cuda):
    S = lib()
    xi = -np.arange(0, 127, dtype=np.float32)
    np.testing.assert_array_equal(_run(S, xi), np.exp2(xi.astype(np.float64)))
    below = np.float32([-126.5, -127.0, -200.0, -1e30, -np.inf])
    np.testing.assert_array_equal(_run(S, below), np.full(below.shape, 2.0 ** -126))


def test_exp2_poly_agrees_with_the_ex2_path(cuda):
    S = lib()
    x = np.linspace(-30.0, 0.0, 100001, dtype=np.float32)
    y = _run(S, x)
    t = torch.exp2(torch.from_numpy(x).cuda()).double().cpu().numpy()
    assert np.max(np.abs(y - t) / t) <= 2.0 ** -21
