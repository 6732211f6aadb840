"""Pins of the oracle's local value pruning (§III.A "Local Value Pruning": after the softmax a head
drops its low-probability V vectors, for this head only).  Reading pinned here: a key's probability
for the head is its column sum over the head's query rows; the head keeps the V vectors of the
v_keep keys ranked first by (higher column sum, lower index); dropped probabilities are not
redistributed; token importance uses the full probabilities, head importance the pruned outputs."""
import numpy as np
import pytest

from oracle import spatten_ref as R


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_keep_all_is_the_plain_head():
    Q, K, V = _rand(1, 6, 4), _rand(2, 9, 4), _rand(3, 9, 4)
    O, P = R.dense_attention(Q, K, V, 0.5)
    O2, P2, kept = R.dense_attention_value_pruned(Q, K, V, 0.5, 9)
    np.testing.assert_array_equal(P2, P)
    np.testing.assert_array_equal(O2, O)
    np.testing.assert_array_equal(kept, np.arange(9))
    kq = R.quantize_head(K.astype(np.float32))
    vq = R.quantize_head(V.astype(np.float32))
    for theta in (0.0, 0.3, 2.0):
        a = R.progressive_attention(Q, kq, vq, theta, 0.5)
        b = R.progressive_attention(Q, kq, vq, theta, 0.5, v_keep=9)
        np.testing.assert_array_equal(a["O"], b["O"])
        np.testing.assert_array_equal(a["P"], b["P"])


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_small(seed):
    n_q, n_kv, d = 5, 7, 3
    Q, K, V = _rand(10 + seed, n_q, d), _rand(20 + seed, n_kv, d), _rand(30 + seed, n_kv, d)
    sm = 0.7
    for v in range(0, n_kv + 1):
        O, P, kept = R.dense_attention_value_pruned(Q, K, V, sm, v)
        # column sums and the ranking written out by hand
        col = [sum(P[i][j] for i in range(n_q)) for j in range(n_kv)]
        want = sorted(sorted(range(n_kv), key=lambda j: (-col[j], j))[:v])
        assert list(kept) == want
        for i in range(n_q):
            for c in range(d):
                ref = sum(P[i][j] * V[j][c] for j in want)
                assert abs(O[i][c] - ref) <= 1e-12 * (1 + abs(ref))


@pytest.mark.parametrize("n,v", [(8, 3), (5, 1), (6, 6), (7, 0)])
def test_uniform_attention_closed_form(n, v):
    """Equal scores: P = 1/n everywhere, every column sum is n_q/n, so the tie rule keeps keys
    0..v-1 and O = (1/n) * sum of their V rows (not 1/v: nothing is renormalised)."""
    n_q, d = 4, 3
    Q, K, V = _rand(5, n_q, d), np.zeros((n, d)), _rand(6, n, d)
    O, P, kept = R.dense_attention_value_pruned(Q, K, V, 1.0, v)
    np.testing.assert_array_equal(kept, np.arange(v))
    want = V[:v].sum(axis=0) / n
    np.testing.assert_allclose(O, np.broadcast_to(want, (n_q, d)), rtol=0, atol=1e-15)


def test_importance_uses_full_probabilities_and_pruned_outputs():
    n, H, d = 6, 2, 4
    Q, K, V = _rand(7, n, H * d), np.zeros((n, H * d)), _rand(8, n, H * d)
    full = R.attention_layer_seq(Q, K, V, [0, 1], d, H, False, 0.0, 1.0)
    pr = R.attention_layer_seq(Q, K, V, [0, 1], d, H, False, 0.0, 1.0, v_keep=2)
    np.testing.assert_array_equal(pr["tok_inc"], full["tok_inc"])     # H * n_q / n per key
    np.testing.assert_allclose(pr["tok_inc"], np.full(n, H * n / n))
    for h in range(H):
        o = V[:2, h * d:(h + 1) * d].sum(axis=0) / n                   # every row of the pruned head
        np.testing.assert_allclose(pr["head_inc"][h], n * np.abs(o).sum(), rtol=1e-13)


def test_dominant_key_survives_alone():
    """One key with a much larger score takes almost all of every row's probability: v_keep = 1
    keeps it and O is (almost) its V row; the other keys' V rows are dropped."""
    n, d = 6, 3
    K = np.zeros((n, d))
    K[4] = [30.0, 0.0, 0.0]
    Q = np.ones((3, d))
    V = _rand(9, n, d)
    O, P, kept = R.dense_attention_value_pruned(Q, K, V, 1.0, 1)
    assert list(kept) == [4]
    np.testing.assert_allclose(O, P[:, [4]] * V[4], rtol=1e-15)
    np.testing.assert_allclose(O, np.broadcast_to(V[4], O.shape), rtol=0, atol=1e-10)


def test_progressive_value_pruning_uses_each_row_precision():
    """theta > 1: every row refetches, so the pruned head is the value-pruned dense head over the
    full 12-bit codes; theta = 0: over the MSB codes.  Keys chosen on the final probabilities."""
    Q, K, V = _rand(11, 5, 4), _rand(12, 9, 4), _rand(13, 9, 4)
    kq, vq = R.quantize_head(K.astype(np.float32)), R.quantize_head(V.astype(np.float32))
    for theta, lsb in ((2.0, True), (0.0, False)):
        Kd = R.dequant(kq["msb"], kq["lsb"] if lsb else None, kq["scale"])
        Vd = R.dequant(vq["msb"], vq["lsb"] if lsb else None, vq["scale"])
        want, _, kept_w = R.dense_attention_value_pruned(Q, Kd, Vd, 0.5, 4)
        r = R.progressive_attention(Q, kq, vq, theta, 0.5, v_keep=4)
        np.testing.assert_array_equal(r["v_kept"], kept_w)
        np.testing.assert_allclose(r["O"], want, rtol=1e-12, atol=1e-14)


def test_decode_step_value_pruning():
    """Decode (one query row per head): keeping every V vector is the plain step; keeping v of
    them gives, per layer and head, the probabilities of the v most probable keys times their V
    rows (checked by hand on the step's own traced projections)."""
    import math
    import test_oracle_cascade as TC
    B, H, d_h, D, T0, L = 2, 2, 8, 16, 20, 2
    _, w_qkv, w_o, caches0 = TC._decode_setup(B, H, d_h, D, T0, L, seed=3)
    x = np.random.default_rng(4).standard_normal((B, D))
    copy = lambda cs: [{k: v.copy() for k, v in c.items()} for c in cs]
    plain = R.decode_step(x, copy(caches0), T0, np.zeros((B, 24)), w_qkv, w_o, H, d_h, lambda n: [n] * L, 2.0)
    same = R.decode_step(x, copy(caches0), T0, np.zeros((B, 24)), w_qkv, w_o, H, d_h, lambda n: [n] * L, 2.0,
                         v_keep_fn=lambda l, k: k)
    np.testing.assert_array_equal(same["x_out"], plain["x_out"])
    caches = copy(caches0)
    v = 5
    r = R.decode_step(x, caches, T0, np.zeros((B, 24)), w_qkv, w_o, H, d_h, lambda n: [n] * L, 2.0,
                      v_keep_fn=lambda l, k: v)
    HD, n = H * d_h, T0 + 1
    xs = r["xs"]
    for l in range(L):
        qkv = xs[l] @ w_qkv[l]
        c = caches[l]
        for b in range(B):
            for h in range(H):
                K = (16.0 * c["k_msb"][b, h, :n] + c["k_lsb"][b, h, :n]) * float(c["k_scale"][b, h])
                V = (16.0 * c["v_msb"][b, h, :n] + c["v_lsb"][b, h, :n]) * float(c["v_scale"][b, h])
                s = (K @ qkv[b, h * d_h:(h + 1) * d_h]) / math.sqrt(d_h)
                p = np.exp(s - s.max())
                p /= p.sum()
                top = sorted(sorted(range(n), key=lambda j: (-p[j], j))[:v])
                want = sum(p[j] * V[j] for j in top)
                np.testing.assert_allclose(r["O"][l][b, h * d_h:(h + 1) * d_h], want, rtol=1e-10, atol=1e-12)
