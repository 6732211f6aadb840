"""Planted mistakes: each mutant replaces one oracle function with a plausible wrong version
(a transposed operand, a dropped term, a wrong sign or rounding or tie rule) and checks that at
least one of the oracle's pins fails.  Mistakes are planted in the oracle only, on the CPU."""
import contextlib
import inspect
import textwrap

import numpy as np
import pytest

from oracle import spatten_ref as R

import test_oracle_attention as TA
import test_oracle_cascade as TC
import test_oracle_quant_topk as TQ
import test_oracle_value_pruning as TV


@contextlib.contextmanager
def patched(name, fn):
    old = getattr(R, name)
    setattr(R, name, fn)
    try:
        yield
    finally:
        setattr(R, name, old)


def _col_softmax(S):
    m = S.max(axis=0, keepdims=True)
    E = np.exp(S - m)
    ell = E.sum(axis=0, keepdims=True)
    return E / ell, ell[0]


def _no_scale_dense(Q, K, V, sm_scale):
    P, _ = R.attention_probs(np.asarray(Q) @ np.asarray(K).T)
    return P @ V, P


def _trunc_split(q):
    q = np.asarray(q, np.int64)
    msb = np.trunc(q / 16).astype(np.int64)
    return msb.astype(np.int8), (q - 16 * msb).astype(np.uint8)


def _swapped_pack(lsb):
    lsb = np.asarray(lsb, np.uint8)
    return (lsb[..., 1::2] | (lsb[..., 0::2] << 4)).astype(np.uint8)


def _scale_2048(x32):
    x = np.asarray(x32, np.float32)
    amax = np.float32(np.max(np.abs(x)))
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(2048))


def _topk_high_index_ties(scores, k):
    s = np.asarray(scores, np.float64)
    n = len(s)
    order = np.lexsort((-np.arange(n), -s))
    return np.sort(order[:k])


def _rowsum_importance(P):
    return np.asarray(P, np.float64).sum(axis=1)


def _signed_head_importance(O):
    return float(np.asarray(O, np.float64).sum())


_orig_prog = R.progressive_attention


def _prog_le(Q, kq, vq, theta, sm_scale, flags_override=None, v_keep=None):
    r = _orig_prog(Q, kq, vq, theta, sm_scale, flags_override, v_keep)
    if flags_override is None:
        fl = r["pmax_msb"] <= theta
        if not np.array_equal(fl, r["flags"]):
            r = _orig_prog(Q, kq, vq, theta, sm_scale, fl, v_keep)
    return r


def _prog_full_v_never(Q, kq, vq, theta, sm_scale, flags_override=None, v_keep=None):
    vq2 = dict(vq, lsb=np.zeros_like(vq["lsb"]))     # forgets the V LSBs on refetch
    return _orig_prog(Q, kq, vq2, theta, sm_scale, flags_override, v_keep)


def source_mutant(fn, old, new):
    """A copy of oracle function `fn` with one statement of its source replaced: a planted mistake
    in a function too large to restate by hand.  The copy calls the unpatched oracle helpers."""
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, old
    ns = dict(vars(R))
    exec(compile(src.replace(old, new), f"<mutant of {fn.__name__}>", "exec"), ns)
    return ns[fn.__name__]


_orig_dequant = R.dequant
_orig_als = R.attention_layer_seq


def _codes_half_away(x32, scale):
    t = np.asarray(x32, np.float32) / np.float32(scale)
    r = np.sign(t) * np.floor(np.abs(t) + np.float32(0.5))     # ties away from zero
    return np.clip(r, -R.QMAX, R.QMAX).astype(np.int32), int(np.count_nonzero(np.abs(r) > R.QMAX))


def _dequant_no_lsb(msb, lsb, scale):
    return _orig_dequant(msb, None, scale)                       # the LSB field is never added


def _unpack_swapped(packed):
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.uint8)
    out[..., 0::2] = p >> 4
    out[..., 1::2] = p & 0xF
    return out


def _gain_on_values(Q, K, V, heads, d_h, H, quant, theta, sm_scale, key_gain=None, flags_override=None,
                    v_keep=None):
    if key_gain is not None:                                     # the boost lands on V, not K
        V = np.asarray(V, np.float64) * np.asarray(key_gain, np.float64)[:, None]
    return _orig_als(Q, K, V, heads, d_h, H, quant, theta, sm_scale, None, flags_override, v_keep)


def _every_head(Q, K, V, heads, d_h, H, quant, theta, sm_scale, key_gain=None, flags_override=None,
                v_keep=None):
    return _orig_als(Q, K, V, range(H), d_h, H, quant, theta, sm_scale, key_gain, flags_override, v_keep)


_cascade_reset_importance = source_mutant(R.cascade_prefill, 'I[b, S] += r["tok_inc"]', 'I[b, S] = r["tok_inc"]')
_cascade_no_residual = source_mutant(R.cascade_prefill, 'X[b, S] = Xk + r["O"] @ w_o[l]', 'X[b, S] = r["O"] @ w_o[l]')
_decode_fresh_scale = source_mutant(   # the appended K row is quantized with its own amax scale
    R.decode_step, 'c["k_msb"][b, h, n_old] = kq["msb"][0]',
    'kq = quantize_head(qkv[b, HD + h * d_h: HD + (h + 1) * d_h][None].astype(np.float32)); '
    'c["k_msb"][b, h, n_old] = kq["msb"][0]')
_decode_keep_old_count = source_mutant(R.decode_step, 'ks = keep_fn(n)', 'ks = keep_fn(n_old)')
_decode_reset_importance = source_mutant(R.decode_step, 'I[b, S] += token_importance_increment(r["P"])',
                                         'I[b, S] = token_importance_increment(r["P"])')


def _vkeep_high_index_ties(P, v_keep):
    P = np.asarray(P, np.float64)
    n = P.shape[1]
    if v_keep is None:
        return np.ones(n), np.arange(n)
    col = P.sum(axis=0)
    kept = np.sort(np.lexsort((-np.arange(n), -col))[:v_keep])   # ties to the higher index
    mask = np.zeros(n)
    mask[kept] = 1.0
    return mask, kept


def _vkeep_by_column_max(P, v_keep):
    P = np.asarray(P, np.float64)
    n = P.shape[1]
    if v_keep is None:
        return np.ones(n), np.arange(n)
    kept = R.topk_select(P.max(axis=0), v_keep)                  # ranks by the largest probability
    mask = np.zeros(n)
    mask[kept] = 1.0
    return mask, kept


MUTANTS = [
    ("attention_probs", _col_softmax, [lambda: TA.test_dense_attention_matches_sdpa(5, 7, 8)]),
    ("dense_attention", _no_scale_dense, [lambda: TA.test_dense_attention_matches_sdpa(5, 7, 8)]),
    ("split_planes", _trunc_split, [TQ.test_quant_codes_golden]),
    ("pack_lsb", _swapped_pack, [TQ.test_lsb_pack_golden]),
    ("quant_scale", _scale_2048, [TQ.test_quant_codes_golden]),
    ("topk_select", _topk_high_index_ties, [lambda: TQ.test_topk_brute_force_small(0), TQ.test_topk_tie_rules]),
    ("token_importance_increment", _rowsum_importance, [TC.test_decode_keep_all_full_equals_dense_over_cache]),
    ("head_importance_increment", _signed_head_importance, [TA.test_head_importance_closed_forms]),
    ("progressive_attention", _prog_le, [lambda: TA.test_constant_keys_refetch_iff_uniform_prob_below_theta(0.1, False)]),
    ("progressive_attention", _prog_full_v_never, [TC.test_cascade_keep_all_always_refetch_equals_dense_on_full_codes]),
    ("value_keep_mask", _vkeep_high_index_ties, [lambda: TV.test_uniform_attention_closed_form(8, 3)]),
    ("value_keep_mask", _vkeep_by_column_max, [lambda s=s: TV.test_brute_force_small(s) for s in range(4)]),
    ("quantize_codes", _codes_half_away, [TQ.test_quant_rounding_brute_force_near_half_boundaries]),
    ("dequant", _dequant_no_lsb, [lambda: TQ.test_quant_identity_and_bounds(0)]),
    ("unpack_lsb", _unpack_swapped, [TQ.test_lsb_pack_golden]),
    ("attention_layer_seq", _gain_on_values, [TA.test_key_gain_scales_key_rows]),
    ("attention_layer_seq", _every_head, [TC.test_cascade_pruning_invariants]),
    ("cascade_prefill", _cascade_reset_importance, [TC.test_cascade_pruning_invariants]),
    ("cascade_prefill", _cascade_no_residual, [TC.test_cascade_keep_all_unquantized_equals_dense_layers]),
    ("decode_step", _decode_fresh_scale, [TC.test_decode_keep_all_full_equals_dense_over_cache]),
    ("decode_step", _decode_keep_old_count, [TC.test_decode_pruning_nested_and_sized]),
    ("decode_step", _decode_reset_importance, [TC.test_decode_keep_all_full_equals_dense_over_cache]),
]


@pytest.mark.parametrize("name,fn,pins", MUTANTS, ids=[f"{m[0]}:{m[1].__name__}" for m in MUTANTS])
def test_pin_catches_planted_mistake(name, fn, pins):
    with patched(name, fn):
        caught = False
        for pin in pins:
            try:
                pin()
            except (AssertionError, ValueError):
                caught = True
        assert caught, f"no pin caught mutant {fn.__name__} of {name}"


def test_importance_increment_closed_form_non_square():
    P = np.array([[0.25, 0.75, 0.0], [0.5, 0.5, 0.0]])
    np.testing.assert_array_equal(R.token_importance_increment(P), [0.75, 1.25, 0.0])
