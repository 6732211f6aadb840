"""Pins for the oracle's quantizer and top-k selection (CPU only).

The quantizer is pinned by hand-derived codes (tests/golden/quant_codes.txt), the identity
q = 16*MSB + LSB, the rounding error bounds and brute force over rounding boundaries.  Top-k is
pinned by brute force over every k-subset (the definition of "the top k under a strict ranking")
and by Python's own sort.
"""
import itertools
import os

import numpy as np
import pytest

from oracle import spatten_ref as R

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_quant_codes_golden():
    rows = _rows("quant_codes.txt")
    x = np.array([float(r[0]) for r in rows], np.float32)
    r = R.quantize_head(x[:, None])
    assert r["scale"] == np.float32(1.0)
    assert r["q"][:, 0].tolist() == [int(r_[1]) for r_ in rows]
    assert r["msb"][:, 0].tolist() == [int(r_[2]) for r_ in rows]
    assert r["lsb"][:, 0].tolist() == [int(r_[3]) for r_ in rows]


def test_lsb_pack_golden():
    with open(os.path.join(GOLD, "lsb_pack.txt")) as f:
        for ln in f:
            if not ln.strip() or ln.startswith("#"):
                continue
            a, b = ln.split("|")
            lsb = np.array([int(t) for t in a.split()], np.uint8)
            packed = np.array([int(t, 16) for t in b.split()], np.uint8)
            np.testing.assert_array_equal(R.pack_lsb(lsb), packed)
            np.testing.assert_array_equal(R.unpack_lsb(packed), lsb)


@pytest.mark.parametrize("seed", range(4))
def test_quant_identity_and_bounds(seed):
    g = np.random.default_rng(seed)
    x = (g.standard_normal((300, 64)) * (10.0 ** g.uniform(-3, 3))).astype(np.float32)
    r = R.quantize_head(x)
    s = float(r["scale"])
    q = r["q"].astype(np.int64)
    assert np.array_equal(16 * r["msb"].astype(np.int64) + r["lsb"], q)
    assert r["msb"].min() >= -128 and r["msb"].max() <= 127
    assert r["lsb"].min() >= 0 and r["lsb"].max() <= 15
    xf = x.astype(np.float64)
    full = R.dequant(r["msb"], r["lsb"], s)
    msb_only = R.dequant(r["msb"], None, s)
    # float32 quotient x/s is rounded once: |x/s - q| <= 1/2 + ulp(2047)/2 = 1/2 + 2**-12
    half = (0.5 + 2.0 ** -12) * s
    assert np.max(np.abs(xf - full)) <= half
    d = xf - msb_only               # zero-filled LSB field: error lies in [-s/2, 15.5 s]
    assert d.min() >= -half and d.max() <= 15.0 * s + half
    # the largest-magnitude element maps to +-2047
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert abs(int(q[i])) == 2047


def test_quant_zero_block_and_saturation():
    r = R.quantize_head(np.zeros((3, 4), np.float32))
    assert r["scale"] == 1.0 and not r["q"].any()
    r = R.quantize_head(np.array([[3000.0, -5000.0, 10.0, 2047.4]], np.float32), scale=1.0)
    assert r["q"][0].tolist() == [2047, -2047, 10, 2047] and r["sat"] == 2


def test_quant_rounding_brute_force_near_half_boundaries():
    # every float32 within a few ulps of j+0.5 (s = 1): round-half-even of the exact quotient
    s = np.float32(1.0)
    for j in range(-40, 40):
        c = np.float32(j + 0.5)
        vals = [c]
        lo = hi = c
        for _ in range(3):
            lo = np.nextafter(lo, np.float32(-np.inf))
            hi = np.nextafter(hi, np.float32(np.inf))
            vals += [lo, hi]
        for v in vals:
            q, _ = R.quantize_codes(np.array([v], np.float32), s)
            exact = float(v)
            if exact == j + 0.5:
                want = j if j % 2 == 0 else j + 1
            else:
                want = int(np.floor(exact + 0.5))
            assert q[0] == want, (v, q[0], want)


def _rank_key(scores, i):
    return (scores[i], -i)          # larger is better: higher score, then lower index


def brute_force_topk(scores, k):
    n = len(scores)
    found = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        worst_in = min((_rank_key(scores, i) for i in sub), default=None)
        best_out = max((_rank_key(scores, i) for i in range(n) if i not in inside), default=None)
        if worst_in is None or best_out is None or worst_in > best_out:
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(25))
def test_topk_brute_force_small(seed):
    g = np.random.default_rng(seed)
    n = int(g.integers(1, 11))
    k = int(g.integers(0, n + 1))
    scores = g.integers(0, 4, size=n).astype(np.float64) * 0.5   # many ties
    if seed % 3 == 0:
        scores[g.integers(0, n)] = -0.0
    got = R.topk_select(scores, k).tolist()
    assert got == brute_force_topk(scores.tolist(), k)


@pytest.mark.parametrize("seed", range(5))
def test_topk_matches_python_sort(seed):
    g = np.random.default_rng(100 + seed)
    n = 2000
    s = np.round(g.lognormal(0, 2, size=n), 1).astype(np.float32).astype(np.float64)
    k = int(g.integers(1, n))
    ref = sorted(range(n), key=lambda i: (-s[i], i))[:k]
    assert R.topk_select(s, k).tolist() == sorted(ref)


def test_topk_tie_rules():
    assert R.topk_select(np.ones(7), 3).tolist() == [0, 1, 2]
    assert R.topk_select(np.array([0.0, -0.0, 0.0, -1.0]), 2).tolist() == [0, 1]
    assert R.topk_select(np.array([1.0, 3.0, 3.0, 2.0]), 1).tolist() == [1]
    with pytest.raises(ValueError):
        R.topk_select(np.array([1.0, np.nan]), 1)
