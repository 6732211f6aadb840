"""GPU parity of spatten_cascade_forward against the oracle.

* float32 tiny cascade (the full workload size): free-running, binding -- kept sets equal (up to
  near-ties within 1e-5 of the k-th score, each logged) and every final row within 1e-4 x RMS
  (against the oracle re-run along the device's kept sets when a near-tie changed one).
* bf16 cascades: layer by layer with the traced device inputs of each layer (teacher forcing, as
  the correctness statement prescribes).  The traced projections used as oracle inputs are
  themselves checked against X_l @ W first (bf16 bound below); the oracle quantizes the traced K
  and V itself (the planes are checked bit-exact in the quantizer tests).  Per layer: O and X_{l+1}
  are the bf16 roundings of values within 2e-2 x RMS of the oracle; token/head selection is
  bit-exact against the oracle run on the device's own importance vectors; against the oracle's
  own importance, kept-set disagreements only at near-ties (1e-5 relative of the k-th score).
"""
import math

import numpy as np
import pytest
import torch

from cascade_token_head_b200 import synth
from oracle import spatten_ref as R

from cascade_helpers import host, run_prefill, upload_prefill
from gpu_helpers import BF, assert_close_bf16_out, assert_close_rms, host_cast, lib

pytestmark = pytest.mark.gpu


def near_tie_ok(scores, got, want, k, rel=1e-5):
    """Disagreeing members of two k-subsets must sit within rel of the k-th largest score."""
    diff = set(got) ^ set(want)
    if not diff:
        return 0
    kth = np.sort(scores)[::-1][k - 1]
    for t in diff:
        assert abs(scores[t] - kth) <= rel * abs(kth), f"kept-set disagreement off a near-tie: {t}"
    print(f"near-tie kept-set disagreements: {len(diff)}")
    return len(diff)


def test_cascade_tiny_fp32_free_running(cuda):
    S = lib()
    w = synth.tiny_fp32()
    d = synth.draw_prefill(w)
    bufs = upload_prefill(S, w, d)
    run_prefill(S, bufs)
    g = host(bufs)
    assert int(g["status"][0]) == 0
    X32 = host_cast(d["X"], torch.float32)
    wq = [host_cast(a, torch.float32) for a in d["w_qkv"]]
    wo = [host_cast(a, torch.float32) for a in d["w_o"]]
    ref = R.cascade_prefill(X32, wq, wo, w.H, w.d_h, w.token_keep, w.head_keep, False, 0.0)
    same = True
    for l in range(w.L):
        k = w.token_keep[l]
        got = g["kept_tok"][l, 0, :k]
        want = ref["kept"][l][0]
        if l > 0:
            near_tie_ok(ref["I_sel"][l - 1][0], got.tolist(), want.tolist(), k)
        assert np.all(np.diff(got) > 0)
        same &= np.array_equal(got, want) and np.array_equal(g["kept_head"][l, 0, :w.head_keep[l]], ref["heads"][l][0])
    # The binding check runs on every final row.  If a near-tie (logged above) made the device keep
    # another token, the oracle is re-run along the device's kept sets, so the rows still compare
    # like for like at 1e-4 x RMS.
    if not same:
        print("near-tie changed a kept set: oracle re-run along the device's selections")
        ref = oracle_along_kept_sets(X32, wq, wo, w, g["kept_tok"][:, 0], g["kept_head"][:, 0])
    assert_close_rms(g["x_out"][0], ref["x_final"][0], 1e-4, "final rows (fp32)")
    np.testing.assert_allclose(g["tok_imp"], ref["I"], rtol=0, atol=1e-5 * ref["I"].max())
    np.testing.assert_allclose(g["head_imp"], ref["J"], rtol=1e-5)


def oracle_along_kept_sets(X, wq, wo, w, kept_tok, kept_head):
    """The oracle's layer step (projection, attention_layer_seq, importance, residual) for one
    sequence, with the token and head sets of every layer taken from the device run instead of
    the oracle's own selection."""
    X = np.array(X[0], np.float64)
    HD = w.H * w.d_h
    I, J = np.zeros(w.T), np.zeros(w.H)
    for l in range(w.L):
        S_l = kept_tok[l, :w.token_keep[l]].astype(np.int64)
        heads = kept_head[l, :w.head_keep[l]].astype(np.int64)
        qkv = X[S_l] @ wq[l]
        r = R.attention_layer_seq(qkv[:, :HD], qkv[:, HD:2 * HD], qkv[:, 2 * HD:], heads, w.d_h, w.H, False, 0.0,
                                  1.0 / math.sqrt(w.d_h))
        I[S_l] += r["tok_inc"]
        J += r["head_inc"]
        X[S_l] = X[S_l] + r["O"] @ wo[l]
    last = kept_tok[w.L - 1, :w.token_keep[-1]].astype(np.int64)
    return dict(x_final=X[last][None], I=I[None], J=J[None])


def teacher_forced_check(S, w, d, sample_b=None):
    """Run the device cascade with traces, then check every layer against the oracle."""
    bufs = upload_prefill(S, w, d)
    run_prefill(S, bufs)
    g = host(bufs)
    assert int(g["status"][0]) == 0
    dt = BF if w.dtype == "bf16" else torch.float32
    HD = w.H * w.d_h
    sm = 1.0 / math.sqrt(w.d_h)
    wq = [host_cast(a, dt) for a in d["w_qkv"]]
    wo = [host_cast(a, dt) for a in d["w_o"]]
    gain = d["key_gain"]
    bs = range(w.B) if sample_b is None else sample_b
    I_ref = np.zeros((w.B, w.T))
    J_ref = np.zeros((w.B, w.H))
    stats = dict(near_tok=0, near_head=0, flag_near=0)
    for l in range(w.L):
        k, Hl = w.token_keep[l], w.head_keep[l]
        for b in bs:
            S_l = g["kept_tok"][l, b, :k].astype(np.int64)
            heads = g["kept_head"][l, b, :Hl].astype(np.int64)
            X_l = g["tx"][l, b, :k].astype(np.float64)
            qkv_dev = g["tqkv"][l, b, :k].astype(np.float64)
            # projections of the device's X_l
            assert_close_bf16_out(qkv_dev, X_l @ wq[l], 2e-2, f"qkv layer {l}")
            gl = None if gain is None else gain[b, S_l].astype(np.float32)
            r = R.attention_layer_seq(qkv_dev[:, :HD], qkv_dev[:, HD:2 * HD], qkv_dev[:, 2 * HD:], heads,
                                      w.d_h, w.H, w.quant, w.theta, sm, key_gain=gl)
            if w.quant:
                dev_flags = {h: g["tflags"][l, b, h, :k].astype(bool) for h in heads}
                fo = {}
                for h in heads:
                    diff = dev_flags[h] != r["flags"][h]
                    if diff.any():
                        assert np.all(np.abs(r["pmax"][h][diff] - w.theta) <= 1e-5 * w.theta), f"flag off a tie, layer {l}"
                        stats["flag_near"] += int(diff.sum())
                    fo[h] = dev_flags[h]
                r = R.attention_layer_seq(qkv_dev[:, :HD], qkv_dev[:, HD:2 * HD], qkv_dev[:, 2 * HD:], heads,
                                          w.d_h, w.H, w.quant, w.theta, sm, key_gain=gl, flags_override=fo)
            O_dev = g["to"][l, b, :k]
            cols = np.concatenate([np.arange(h * w.d_h, (h + 1) * w.d_h) for h in heads])
            assert_close_bf16_out(O_dev[:, cols], r["O"][:, cols], 2e-2, f"O layer {l}")
            I_ref[b, S_l] += r["tok_inc"]
            J_ref[b] += r["head_inc"]
            # device importance after layer l against the teacher-forced oracle importance
            np.testing.assert_allclose(g["ttok"][l, b], I_ref[b], rtol=0, atol=2e-5 * I_ref[b].max() + 1e-7)
            np.testing.assert_allclose(g["thead"][l, b], J_ref[b], rtol=2e-2)
            if l == w.L - 1:
                X_next_ref = X_l + O_dev.astype(np.float64) @ wo[l]
                assert_close_bf16_out(g["x_out"][b], X_next_ref, 2e-2, "final rows")
                continue
            k2, H2 = w.token_keep[l + 1], w.head_keep[l + 1]
            S_n = g["kept_tok"][l + 1, b, :k2].astype(np.int64)
            # bit-exact selection on the device's own importance
            dev_I = g["ttok"][l, b].astype(np.float64)
            np.testing.assert_array_equal(S_n, S_l[R.topk_select(dev_I[S_l], k2)])
            # against the oracle's importance: only near-ties may differ
            want = S_l[R.topk_select(I_ref[b, S_l], k2)]
            stats["near_tok"] += _near(I_ref[b, S_l], S_l, S_n, want, k2)
            H_n = g["kept_head"][l + 1, b, :H2].astype(np.int64)
            dev_J = g["thead"][l, b].astype(np.float64)
            np.testing.assert_array_equal(H_n, heads[R.topk_select(dev_J[heads], H2)])
            # next layer's rows: the kept rows of X_l + O W_o
            X_next_ref = X_l + O_dev.astype(np.float64) @ wo[l]
            pos = np.searchsorted(S_l, S_n)
            assert_close_bf16_out(g["tx"][l + 1, b, :k2], X_next_ref[pos], 2e-2, f"X layer {l + 1}")
    return stats


def _near(scores_on_S, S_l, got, want, k):
    diff = set(got.tolist()) ^ set(want.tolist())
    if not diff:
        return 0
    kth = np.sort(scores_on_S)[::-1][k - 1]
    lookup = dict(zip(S_l.tolist(), scores_on_S.tolist()))
    for t in diff:
        assert abs(lookup[t] - kth) <= 1e-5 * abs(kth), f"kept-set disagreement off a near-tie: token {t}"
    return len(diff)


@pytest.mark.parametrize("B,T,L,d_h,H", [(2, 96, 4, 64, 4), (2, 257, 5, 64, 6), (1, 300, 3, 128, 4)])
def test_cascade_bf16_small_teacher_forced(cuda, B, T, L, d_h, H):
    S = lib()
    from fractions import Fraction
    w = synth.PrefillWorkload("small", B=B, T=T, D=H * d_h, H=H, d_h=d_h, L=L, dtype="bf16",
                              token_keep=synth.geometric_keep(T, Fraction(4, 5), L),
                              head_keep=[H] + [max(1, H - (l + 1) // 2) for l in range(1, L)],
                              quant=True, theta=0.1, boost=("uniform", max(1, T // 20), 4.0))
    d = synth.draw_prefill(w)
    stats = teacher_forced_check(S, w, d)
    print(stats)


def test_cascade_bert_full_size_sampled(cuda):
    """The BERT-base prefill workload at full size; sequences 0 and 17 checked layer by layer."""
    S = lib()
    w = synth.bert_base_prefill()
    d = synth.draw_prefill(w)
    stats = teacher_forced_check(S, w, d, sample_b=[0, 17])
    print(stats)


def test_cascade_deterministic(cuda):
    S = lib()
    from fractions import Fraction
    w = synth.PrefillWorkload("det", B=4, T=256, D=768, H=12, d_h=64, L=4, dtype="bf16",
                              token_keep=synth.geometric_keep(256, Fraction(9, 10), 4), head_keep=[12, 12, 11, 11],
                              quant=True, theta=0.1, boost=("uniform", 13, 4.0))
    d = synth.draw_prefill(w)
    a = upload_prefill(S, w, d, trace=False)
    run_prefill(S, a)
    ha = host(a)
    run_prefill(S, a)
    hb = host(a)
    for key in ("x_out", "kept_tok", "kept_head", "tok_imp", "head_imp", "refetch"):
        np.testing.assert_array_equal(ha[key], hb[key])


def test_cascade_untraced_equals_traced(cuda):
    """Without traces the importance reduction and the next layer's selections run on the
    library's second stream, beside the output projection; with traces they stay on the caller's
    stream.  Both orders give bit-identical results (the same kernels in the same data order)."""
    S = lib()
    from fractions import Fraction
    w = synth.PrefillWorkload("side", B=4, T=256, D=768, H=12, d_h=64, L=5, dtype="bf16",
                              token_keep=synth.geometric_keep(256, Fraction(9, 10), 5), head_keep=[12, 12, 11, 11, 10],
                              quant=True, theta=0.1, boost=("uniform", 13, 4.0))
    d = synth.draw_prefill(w)
    a = upload_prefill(S, w, d, trace=False)
    run_prefill(S, a)
    plain = host(a)
    t = upload_prefill(S, w, d, trace=True)
    run_prefill(S, t)
    traced = host(t)
    for key in ("x_out", "kept_tok", "kept_head", "tok_imp", "head_imp", "refetch"):
        np.testing.assert_array_equal(plain[key], traced[key])
