"""Pins for the oracle's cascade (prefill) and decode step (CPU only).

With every token and head kept and the LSBs always fetched, the cascade must equal a plain
layer loop of dense attention (torch float64 SDPA) on the full-precision K/V; kept sets must be
nested with the scheduled sizes; importance must sum to queries x heads per layer.
"""
import math
import os

import numpy as np
import pytest
import torch

from cascade_token_head_b200 import synth
from oracle import spatten_ref as R

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def sdpa64(Q, K, V, scale):
    q, k, v = (torch.tensor(np.asarray(a, np.float64))[None, None] for a in (Q, K, V))
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)[0, 0].numpy()


def small_prefill(**over):
    base = dict(name="t", B=2, T=48, D=32, H=4, d_h=8, L=3, dtype="f32",
                token_keep=[48, 48, 48], head_keep=[4, 4, 4], quant=False, theta=0.0, boost=None)
    base.update(over)
    return synth.PrefillWorkload(**base)


def test_keep_schedules_golden():
    want = {}
    with open(os.path.join(GOLD, "keep_schedules.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                key, vals = ln.split(":")
                want[key.strip()] = [int(v) for v in vals.split()]
    assert synth.tiny_fp32().token_keep == want["tiny_cascade_fp32 tokens"]
    assert synth.bert_base_prefill().token_keep == want["bert_base_prefill_bf16 tokens"]
    assert synth.bert_base_prefill().head_keep == want["bert_base_prefill_bf16 heads"]
    assert synth.long_prefill().token_keep == want["long_context_prefill_bf16 tokens"]
    assert synth.long_prefill().head_keep == want["long_context_prefill_bf16 heads"]
    assert synth.linear_decode_keep(1025, 24)[:3] == want["gpt2_medium_decode n=1025 first3"]
    assert synth.linear_decode_keep(1025, 24)[-1] == want["gpt2_medium_decode n=1025 last"][0]
    assert synth.linear_decode_keep(1152, 24)[-1] == want["gpt2_medium_decode n=1152 last"][0]


def _plain_layers(X, w_qkv, w_o, H, d_h, K_transform=None):
    """Independent reference: X <- X + concat_h SDPA(Q_h, K_h, V_h) W_o, all tokens and heads."""
    X = np.array(X, np.float64)
    HD = H * d_h
    for l in range(len(w_qkv)):
        for b in range(X.shape[0]):
            qkv = X[b] @ w_qkv[l]
            O = np.zeros((X.shape[1], HD))
            for h in range(H):
                sl = slice(h * d_h, (h + 1) * d_h)
                Q, K, V = qkv[:, sl], qkv[:, HD:][:, sl], qkv[:, 2 * HD:][:, sl]
                if K_transform is not None:
                    K, V = K_transform(K), K_transform(V)
                O[:, sl] = sdpa64(Q, K, V, 1.0 / math.sqrt(d_h))
            X[b] = X[b] + O @ w_o[l]
    return X


def test_cascade_keep_all_unquantized_equals_dense_layers():
    w = small_prefill()
    d = synth.draw_prefill(w)
    r = R.cascade_prefill(d["X"], d["w_qkv"], d["w_o"], w.H, w.d_h, w.token_keep, w.head_keep,
                          False, 0.0)
    ref = _plain_layers(d["X"], d["w_qkv"], d["w_o"], w.H, w.d_h)
    np.testing.assert_allclose(r["X"], ref, rtol=1e-11, atol=1e-11)


def test_cascade_keep_all_always_refetch_equals_dense_on_full_codes():
    w = small_prefill(quant=True, theta=2.0)
    d = synth.draw_prefill(w)
    r = R.cascade_prefill(d["X"], d["w_qkv"], d["w_o"], w.H, w.d_h, w.token_keep, w.head_keep,
                          True, 2.0)

    def full_codes(M):                     # 12-bit round trip, written out independently
        m32 = M.astype(np.float32)
        amax = np.float32(np.abs(m32).max())
        s = np.float32(amax / np.float32(2047))
        q = np.clip(np.rint(m32 / s), -2047, 2047)
        return q.astype(np.float64) * float(s)

    ref = _plain_layers(d["X"], d["w_qkv"], d["w_o"], w.H, w.d_h, K_transform=full_codes)
    np.testing.assert_allclose(r["X"], ref, rtol=1e-10, atol=1e-10)
    assert r["refetch"] == [w.B * w.T * w.H] * w.L


def test_cascade_pruning_invariants():
    w = small_prefill(B=3, T=40, L=4, token_keep=[40, 30, 22, 17], head_keep=[4, 4, 3, 2],
                      quant=True, theta=0.2, boost=("uniform", 3, 4.0))
    d = synth.draw_prefill(w)
    r = R.cascade_prefill(d["X"], d["w_qkv"], d["w_o"], w.H, w.d_h, w.token_keep, w.head_keep,
                          True, 0.2, key_gain=d["key_gain"])
    for b in range(w.B):
        prev_t, prev_h = set(range(w.T)), set(range(w.H))
        for l in range(w.L):
            S, Hs = r["kept"][l][b], r["heads"][l][b]
            assert len(S) == w.token_keep[l] and len(Hs) == w.head_keep[l]
            assert list(S) == sorted(S) and set(S) <= prev_t and set(Hs) <= prev_h
            prev_t, prev_h = set(S), set(Hs)
        # importance sums to sum_l (queries x kept heads)
        total = sum(w.token_keep[l] * w.head_keep[l] for l in range(w.L))
        np.testing.assert_allclose(r["I"][b].sum(), total, rtol=1e-12)
        # pruned rows of X are frozen at the value they had when pruned
        last = set(r["kept"][-1][b])
        dropped = [t for t in range(w.T) if t not in last]
        assert len(dropped) == w.T - w.token_keep[-1]
    assert r["x_final"].shape == (w.B, w.token_keep[-1], w.D)


def test_cascade_selection_follows_cumulative_importance():
    # after layer 0, the kept set is the top-k of I over all tokens (ties to lower index)
    w = small_prefill(B=1, T=30, L=2, token_keep=[30, 11], head_keep=[4, 4])
    d = synth.draw_prefill(w)
    r1 = R.cascade_prefill(d["X"], d["w_qkv"][:1], d["w_o"][:1], w.H, w.d_h, [30], [4], False, 0.0)
    I0 = r1["I"][0]
    order = sorted(range(30), key=lambda i: (-I0[i], i))[:11]
    r2 = R.cascade_prefill(d["X"], d["w_qkv"], d["w_o"], w.H, w.d_h, w.token_keep, w.head_keep,
                           False, 0.0)
    assert r2["kept"][1][0].tolist() == sorted(order)


def _decode_setup(B=2, H=2, d_h=8, D=16, T0=20, L=3, cap=24, seed=0):
    g = np.random.default_rng(seed)
    w_qkv = [g.standard_normal((D, 3 * H * d_h)) / math.sqrt(D) for _ in range(L)]
    w_o = [g.standard_normal((H * d_h, D)) / math.sqrt(D) for _ in range(L)]
    caches = R.empty_decode_caches(L, B, H, cap, d_h)
    for l in range(L):
        R.quantize_prompt_cache(caches[l], g.standard_normal((B, H, T0, d_h)).astype(np.float32),
                                g.standard_normal((B, H, T0, d_h)).astype(np.float32))
    return g, w_qkv, w_o, caches


def test_decode_keep_all_full_equals_dense_over_cache():
    B, H, d_h, D, T0, L = 2, 2, 8, 16, 20, 3
    g, w_qkv, w_o, caches = _decode_setup(B, H, d_h, D, T0, L)
    x = g.standard_normal((B, D))
    I = np.zeros((B, 24))
    before = [{k: v.copy() for k, v in c.items()} for c in caches]
    r = R.decode_step(x, caches, T0, I, w_qkv, w_o, H, d_h, lambda n: [n] * L, theta=2.0)
    xr = x.copy()
    HD = H * d_h
    for l in range(L):
        qkv = xr @ w_qkv[l]
        O = np.zeros((B, HD))
        for b in range(B):
            for h in range(H):
                c = before[l]
                sk, sv = float(c["k_scale"][b, h]), float(c["v_scale"][b, h])
                kn = np.clip(np.rint(qkv[b, HD + h * d_h:HD + (h + 1) * d_h].astype(np.float32) / np.float32(sk)), -2047, 2047)
                vn = np.clip(np.rint(qkv[b, 2 * HD + h * d_h:2 * HD + (h + 1) * d_h].astype(np.float32) / np.float32(sv)), -2047, 2047)
                Kc = (16.0 * c["k_msb"][b, h, :T0] + c["k_lsb"][b, h, :T0]) * sk
                Vc = (16.0 * c["v_msb"][b, h, :T0] + c["v_lsb"][b, h, :T0]) * sv
                K = np.vstack([Kc, kn.astype(np.float64) * sk])
                V = np.vstack([Vc, vn.astype(np.float64) * sv])
                O[b, h * d_h:(h + 1) * d_h] = sdpa64(qkv[b, h * d_h:(h + 1) * d_h][None], K, V,
                                                     1 / math.sqrt(d_h))[0]
        np.testing.assert_allclose(r["O"][l], O, rtol=1e-10, atol=1e-12)
        xr = xr + O @ w_o[l]
    np.testing.assert_allclose(r["x_out"], xr, rtol=1e-10, atol=1e-12)
    # one query per head per layer: importance sums to H * L per sequence
    np.testing.assert_allclose(I.sum(1), H * L, rtol=1e-12)
    assert np.all(I[:, T0 + 1:] == 0)


def test_decode_pruning_nested_and_sized():
    B, H, d_h, D, T0, L = 2, 2, 8, 16, 20, 4
    g, w_qkv, w_o, caches = _decode_setup(B, H, d_h, D, T0, L, cap=26)
    I = np.zeros((B, 26))
    for step in range(3):
        n_old = T0 + step
        r = R.decode_step(g.standard_normal((B, D)), caches, n_old, I, w_qkv, w_o, H, d_h,
                          lambda n: synth.linear_decode_keep(n, L), theta=0.2)
        ks = synth.linear_decode_keep(n_old + 1, L)
        for b in range(B):
            prev = set(range(n_old + 1))
            for l in range(L):
                S = r["kept"][l][b]
                assert len(S) == ks[l] and set(S) <= prev and list(S) == sorted(S)
                prev = set(S)
