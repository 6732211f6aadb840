"""Pins for the oracle's attention, progressive quantization and importance (CPU only).

Each check compares the oracle with something other than itself: torch's float64
scaled_dot_product_attention (a library routine), a hand-written triple loop, closed forms and
invariants that follow from the definitions in SpAtten §II and §IV.E.
"""
import math

import numpy as np
import pytest
import torch

from oracle import spatten_ref as R


def sdpa64(Q, K, V, scale):
    q = torch.tensor(np.asarray(Q, np.float64))[None, None]
    k = torch.tensor(np.asarray(K, np.float64))[None, None]
    v = torch.tensor(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)[0, 0].numpy()


def triple_loop_attention(Q, K, V, scale):
    nq, nk, dv = len(Q), len(K), len(V[0])
    out = [[0.0] * dv for _ in range(nq)]
    for i in range(nq):
        s = [sum(Q[i][d] * K[j][d] for d in range(len(Q[i]))) * scale for j in range(nk)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        for d in range(dv):
            out[i][d] = sum(e[j] / z * V[j][d] for j in range(nk))
    return np.array(out)


@pytest.mark.parametrize("nq,nk,d", [(1, 1, 4), (5, 7, 8), (33, 65, 64), (17, 200, 128)])
def test_dense_attention_matches_sdpa(nq, nk, d):
    g = np.random.default_rng(nq * 1000 + nk)
    Q, K, V = g.standard_normal((nq, d)), g.standard_normal((nk, d)), g.standard_normal((nk, d))
    scale = 1.0 / math.sqrt(d)
    O, P = R.dense_attention(Q, K, V, scale)
    np.testing.assert_allclose(O, sdpa64(Q, K, V, scale), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=1e-14)


def test_dense_attention_matches_triple_loop():
    g = np.random.default_rng(7)
    Q, K, V = g.standard_normal((4, 3)), g.standard_normal((6, 3)), g.standard_normal((6, 2))
    O, _ = R.dense_attention(Q, K, V, 0.5)
    np.testing.assert_allclose(O, triple_loop_attention(Q.tolist(), K.tolist(), V.tolist(), 0.5),
                               rtol=1e-12)


def test_probs_closed_form():
    # scores [0, log 3] -> probabilities [1/4, 3/4]; ell = 1 + 1/3 and max prob = 1/ell
    P, ell = R.attention_probs(np.array([[0.0, math.log(3.0)]]))
    np.testing.assert_allclose(P, [[0.25, 0.75]], rtol=1e-15)
    np.testing.assert_allclose(ell, [4.0 / 3.0], rtol=1e-15)
    np.testing.assert_allclose(1.0 / ell, P.max(1), rtol=1e-15)


def _block(g, n, d, boost_rows=()):
    x = g.standard_normal((n, d)).astype(np.float32)
    for r in boost_rows:
        x[r] *= 4
    return x


def test_progressive_theta_zero_is_msb_attention():
    g = np.random.default_rng(1)
    n, d = 40, 64
    Q = g.standard_normal((n, d))
    kq, vq = R.quantize_head(_block(g, n, d)), R.quantize_head(_block(g, n, d))
    r = R.progressive_attention(Q, kq, vq, 0.0, 1 / 8)
    assert not r["flags"].any()
    Km = kq["scale"] * 16.0 * kq["msb"].astype(np.float64)
    Vm = vq["scale"] * 16.0 * vq["msb"].astype(np.float64)
    np.testing.assert_allclose(r["O"], sdpa64(Q, Km, Vm, 1 / 8), rtol=1e-11, atol=1e-13)


def test_progressive_theta_above_one_is_full_attention():
    g = np.random.default_rng(2)
    n, d = 40, 64
    Q = g.standard_normal((n, d))
    kq, vq = R.quantize_head(_block(g, n, d)), R.quantize_head(_block(g, n, d))
    r = R.progressive_attention(Q, kq, vq, 2.0, 1 / 8)
    assert r["flags"].all()
    Kf = kq["scale"] * kq["q"].astype(np.float64)
    Vf = vq["scale"] * vq["q"].astype(np.float64)
    np.testing.assert_allclose(r["O"], sdpa64(Q, Kf, Vf, 1 / 8), rtol=1e-11, atol=1e-13)


def test_progressive_mixed_rows_follow_their_own_precision():
    g = np.random.default_rng(3)
    n, d = 64, 64
    Q = g.standard_normal((n, d)) * np.where(np.arange(n) % 2 == 0, 4.0, 0.2)[:, None]
    kq, vq = R.quantize_head(_block(g, n, d)), R.quantize_head(_block(g, n, d))
    r = R.progressive_attention(Q, kq, vq, 0.1, 1 / 8)
    assert 0 < r["flags"].sum() < n
    Km = kq["scale"] * 16.0 * kq["msb"].astype(np.float64)
    Vm = vq["scale"] * 16.0 * vq["msb"].astype(np.float64)
    Kf = kq["scale"] * kq["q"].astype(np.float64)
    Vf = vq["scale"] * vq["q"].astype(np.float64)
    O_m, O_f = sdpa64(Q, Km, Vm, 1 / 8), sdpa64(Q, Kf, Vf, 1 / 8)
    # the decision uses the MSB-pass max probability, computed here independently
    S = Q @ Km.T / 8
    pmax = np.exp(S.max(1) - S.max(1)) / np.exp(S - S.max(1, keepdims=True)).sum(1)
    np.testing.assert_array_equal(r["flags"], pmax < 0.1)
    for i in range(n):
        np.testing.assert_allclose(r["O"][i], O_f[i] if r["flags"][i] else O_m[i], rtol=1e-10,
                                   atol=1e-12)


def test_single_key_never_refetches():
    g = np.random.default_rng(4)
    Q = g.standard_normal((9, 8))
    kq, vq = R.quantize_head(_block(g, 1, 8)), R.quantize_head(_block(g, 1, 8))
    r = R.progressive_attention(Q, kq, vq, 0.999, 0.5)
    assert not r["flags"].any()
    np.testing.assert_allclose(r["P"], 1.0)


@pytest.mark.parametrize("theta,expect", [(0.1, False), (0.1000001, True), (0.05, False)])
def test_constant_keys_refetch_iff_uniform_prob_below_theta(theta, expect):
    # 10 identical keys: every row is uniform, max prob = 1/10 exactly; strict comparison
    g = np.random.default_rng(5)
    k = np.tile(g.standard_normal((1, 16)).astype(np.float32), (10, 1))
    Q = g.standard_normal((3, 16))
    kq, vq = R.quantize_head(k), R.quantize_head(_block(g, 10, 16))
    r = R.progressive_attention(Q, kq, vq, theta, 0.25)
    assert r["flags"].tolist() == [expect] * 3
    np.testing.assert_allclose(r["P"], 0.1, rtol=1e-14)


def test_token_importance_sums_to_queries_times_heads():
    g = np.random.default_rng(6)
    n, H, d = 37, 3, 16
    Q, K, V = (g.standard_normal((n, H * d)) for _ in range(3))
    r = R.attention_layer_seq(Q, K, V, [0, 2], d, H, quant=True, theta=0.3, sm_scale=0.25)
    np.testing.assert_allclose(r["tok_inc"].sum(), n * 2, rtol=1e-12)
    assert r["head_inc"][1] == 0.0 and np.all(r["O"][:, d:2 * d] == 0)


def test_identical_keys_give_uniform_importance():
    g = np.random.default_rng(8)
    n, H, d = 12, 2, 8
    Q, V = g.standard_normal((n, H * d)), g.standard_normal((n, H * d))
    K = np.tile(g.standard_normal((1, H * d)), (n, 1))
    r = R.attention_layer_seq(Q, K, V, [0, 1], d, H, quant=False, theta=0.0, sm_scale=0.3)
    np.testing.assert_allclose(r["tok_inc"], np.full(n, n * H / n), rtol=1e-13)


def test_head_importance_closed_forms():
    g = np.random.default_rng(9)
    n, d = 20, 8
    Q, K, V = g.standard_normal((n, d)), g.standard_normal((n, d)), g.standard_normal((n, d))
    r0 = R.attention_layer_seq(Q, K, 0 * V, [0], d, 1, False, 0.0, 0.3)
    assert r0["head_inc"][0] == 0.0
    r1 = R.attention_layer_seq(Q, K, V, [0], d, 1, False, 0.0, 0.3)
    r2 = R.attention_layer_seq(Q, K, -3.0 * V, [0], d, 1, False, 0.0, 0.3)
    np.testing.assert_allclose(r2["head_inc"][0], 3.0 * r1["head_inc"][0], rtol=1e-13)
    # one key: every output row is that key's value vector
    r3 = R.attention_layer_seq(Q, K[:1], V[:1], [0], d, 1, False, 0.0, 0.3)
    np.testing.assert_allclose(r3["head_inc"][0], n * np.abs(V[0]).sum(), rtol=1e-13)


def test_key_gain_scales_key_rows():
    # gain g on key j is the same as multiplying K[j] by g before attention
    g = np.random.default_rng(10)
    n, d = 10, 8
    Q, K, V = g.standard_normal((n, d)), g.standard_normal((n, d)), g.standard_normal((n, d))
    gain = np.ones(n)
    gain[[2, 7]] = 4.0
    r = R.attention_layer_seq(Q, K, V, [0], d, 1, False, 0.0, 0.3, key_gain=gain)
    np.testing.assert_allclose(r["O"], sdpa64(Q, K * gain[:, None], V, 0.3), rtol=1e-12)
