"""Oracle for SpAtten cascade token/head pruning with progressive quantization.

TEST INFRASTRUCTURE ONLY.  This is a plain, slow, float64 CPU restatement of what the hot path
computes.  Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it.  It shares no code with the CUDA library (no kernels, headers, helpers or tables) and
imports nothing from it; both sides only read inputs from the seeded generators.

Source: "SpAtten: Efficient Sparse Attention Architecture with Cascade Token and Head Pruning"
(Wang, Zhang, Han; arXiv 2012.09852v3), as summarised on its paperlayer.ai page.  Section names
below are that page's: §II "Background and Motivation", §II.B "Motivation", §III.A "Cascade Token
Pruning" (printed as "A." after §II.B), §IV "Hardware Architecture", §IV.B "Top-k Engine",
§IV.E "Query-Key Multiplication Module".

Readings where the page is silent:
  * scale is 1/sqrt(d_h) ("scaled Q x K^T", §II);
  * 12-bit symmetric codes, one float32 scale per (sequence, layer, head, tensor) computed as
    amax/2047 in float32; codes are round-half-even of float32(x)/s, clamped to +-2047;
    MSB = floor(q/16) (int8), LSB = q - 16*MSB (0..15); MSB-only values zero-fill the LSB field;
  * V is progressive too, with the same per-row decision as K ("recomputes the attention outputs");
  * the refetch test uses the MSB-pass probabilities: refetch iff max_j p_ij < theta (strict), so
    theta <= 0 never refetches and theta > 1 always does; importance uses the final probabilities;
  * token importance accumulates the column sums of the final probabilities over every kept head,
    query and layer (and decode step); head importance accumulates sum |O_h| before W_o;
  * selection ranks by (higher score, then lower index) and returns indices in ascending order;
  * layers are attention-only with a residual: X_kept += concat_h(O_h) @ W_o, pruned heads give 0.

Parity pins: every public function here is pinned by a CPU test against something other than
itself (library routines, closed forms, invariants, brute force); see tests/test_oracle_*.py.
"""
from __future__ import annotations

import math

import numpy as np

QMAX = 2047          # largest 12-bit symmetric code
LSB_BITS = 4         # width of the LSB plane (8-bit MSB + 4-bit LSB)


# ---------------------------------------------------------------------------------------------
# C1  dense attention for one head (SpAtten §II "Attention mechanism")
# ---------------------------------------------------------------------------------------------
def attention_probs(S: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Row softmax of a score matrix, computed as exp(S - rowmax) / sum.  Returns (P, ell) where
    ell_i = sum_j exp(s_ij - max_j s_ij), so that max_j p_ij = 1/ell_i."""
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    ell = E.sum(axis=1, keepdims=True)
    return E / ell, ell[:, 0]


def dense_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, sm_scale: float):
    """One head: S = Q K^T * scale, P = row-softmax(S), O = P V.  No mask (summarization is
    bidirectional, §II "Attention-based NLP models").  Returns (O, P)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    S = (Q @ K.T) * sm_scale
    P, _ = attention_probs(S)
    return P @ V, P


# ---------------------------------------------------------------------------------------------
# C2  progressive quantization planes (§III.A "Progressive Quantization", §IV "Quantization
#     Support": MSBs and LSBs are fetched separately and concatenated by a bitwidth converter)
# ---------------------------------------------------------------------------------------------
def quant_scale(x32: np.ndarray) -> np.float32:
    """float32 scale s = amax / 2047 over all elements; s = 1 when amax == 0."""
    x = np.asarray(x32, np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(QMAX))


def quantize_codes(x32: np.ndarray, scale) -> tuple[np.ndarray, int]:
    """12-bit codes q = clamp(rint_half_even(float32(x) / s), -2047, 2047) in float32 division.
    Returns (q int32, number of saturated elements)."""
    x = np.asarray(x32, np.float32)
    s = np.float32(scale)
    r = np.rint(x / s)                       # float32 / float32 -> float32, IEEE round-to-nearest
    sat = int(np.count_nonzero(np.abs(r) > QMAX))
    q = np.clip(r, -QMAX, QMAX).astype(np.int32)
    return q, sat


def split_planes(q: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """MSB = floor(q / 16) as int8 in [-128, 127]; LSB = q - 16*MSB in [0, 15]."""
    q = np.asarray(q, np.int64)
    msb = np.floor_divide(q, 1 << LSB_BITS)
    lsb = q - (msb << LSB_BITS)
    return msb.astype(np.int8), lsb.astype(np.uint8)


def pack_lsb(lsb: np.ndarray) -> np.ndarray:
    """Pack a [..., d] LSB plane two nibbles per byte: element 2c in bits 0-3, 2c+1 in bits 4-7."""
    lsb = np.asarray(lsb, np.uint8)
    lo = lsb[..., 0::2]
    hi = lsb[..., 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_lsb(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def quantize_head(x32: np.ndarray, scale=None):
    """Quantize one (sequence, head, tensor) block [n, d_h].  With scale=None the scale is the
    block's amax/2047; otherwise the given (prompt-time) scale is used and saturations counted.
    Returns dict(msb, lsb (unpacked), scale, q, sat)."""
    s = quant_scale(x32) if scale is None else np.float32(scale)
    q, sat = quantize_codes(x32, s)
    msb, lsb = split_planes(q)
    return dict(msb=msb, lsb=lsb, scale=s, q=q, sat=sat)


def dequant(msb: np.ndarray, lsb: np.ndarray | None, scale) -> np.ndarray:
    """x_hat = s * (16*MSB + LSB); with lsb=None the LSB field is zero-filled (MSB-only)."""
    v = np.asarray(msb, np.float64) * (1 << LSB_BITS)
    if lsb is not None:
        v = v + np.asarray(lsb, np.float64)
    return float(scale) * v


# ---------------------------------------------------------------------------------------------
# C3  progressive-quantization attention for one head (§IV.E "Progressive Quantization")
# ---------------------------------------------------------------------------------------------
def progressive_attention(Q, kq: dict, vq: dict, theta: float, sm_scale: float,
                          flags_override: np.ndarray | None = None, v_keep: int | None = None):
    """MSB pass first; rows whose max probability is below theta refetch the LSBs and recompute
    their scores, probabilities and outputs with the full 12-bit K and V.

    ``kq``/``vq`` are quantize_head() results.  ``flags_override`` (bool [n_q]) replaces the
    computed decision; it is used only to compare against a device run row by row after the
    near-tie rows were checked.  ``v_keep``: local value pruning of this head (see
    value_keep_mask) on the final probabilities; None keeps every V vector.
    Returns dict(O, P, flags, pmax_msb, v_kept).
    """
    Q = np.asarray(Q, np.float64)
    K_msb = dequant(kq["msb"], None, kq["scale"])
    V_msb = dequant(vq["msb"], None, vq["scale"])
    S_msb = (Q @ K_msb.T) * sm_scale
    P_msb, ell = attention_probs(S_msb)
    pmax = 1.0 / ell
    flags = pmax < theta
    if flags_override is not None:
        flags = np.asarray(flags_override, bool)
    P = P_msb.copy()
    rows = np.nonzero(flags)[0]
    if rows.size:
        K_full = dequant(kq["msb"], kq["lsb"], kq["scale"])
        S_full = (Q[rows] @ K_full.T) * sm_scale
        P_full, _ = attention_probs(S_full)
        P[rows] = P_full
    mask, kept = value_keep_mask(P, v_keep)
    Pv = P * mask                      # P itself when every V vector is kept
    O = Pv @ V_msb
    if rows.size:
        V_full = dequant(vq["msb"], vq["lsb"], vq["scale"])
        O[rows] = Pv[rows] @ V_full
    return dict(O=O, P=P, flags=flags, pmax_msb=pmax, v_kept=kept)


# ---------------------------------------------------------------------------------------------
# local value pruning (§III.A "Local Value Pruning")
# ---------------------------------------------------------------------------------------------
def value_keep_mask(P: np.ndarray, v_keep: int | None):
    """After the softmax a head drops its low-probability V vectors, for this head only (nothing
    is removed from other heads or layers).  Reading: a key's probability for the head is its
    column sum over the head's query rows (its share of the head's attention; one query row in
    decode); the head keeps the V vectors of the v_keep keys ranked first by (higher column sum,
    then lower index), the top-k rule; the dropped keys' probabilities are not redistributed.
    Returns (mask [n_kv] of 0/1 floats, kept indices ascending); v_keep None keeps all."""
    P = np.asarray(P, np.float64)
    n = P.shape[1]
    if v_keep is None:
        return np.ones(n), np.arange(n)
    kept = topk_select(P.sum(axis=0), int(v_keep))
    mask = np.zeros(n)
    mask[kept] = 1.0
    return mask, kept


def dense_attention_value_pruned(Q, K, V, sm_scale: float, v_keep: int | None):
    """C1 followed by local value pruning of the head: O = (P * mask) @ V."""
    O, P = dense_attention(Q, K, V, sm_scale)
    if v_keep is None:
        return O, P, np.arange(P.shape[1])
    mask, kept = value_keep_mask(P, v_keep)
    return (P * mask) @ np.asarray(V, np.float64), P, kept


# ---------------------------------------------------------------------------------------------
# C4/C5  importance increments (§II "Cascade pruning", §II.B "Token pruning", §III.A)
# ---------------------------------------------------------------------------------------------
def token_importance_increment(P: np.ndarray) -> np.ndarray:
    """Column sum of one head's probabilities: how much attention every key token received."""
    return np.asarray(P, np.float64).sum(axis=0)


def head_importance_increment(O: np.ndarray) -> float:
    """Sum of absolute attention-output values of one head."""
    return float(np.abs(np.asarray(O, np.float64)).sum())


# ---------------------------------------------------------------------------------------------
# C7  top-k selection (§II "Cascade pruning": keep the top-k by the pruning ratio; §IV.B)
# ---------------------------------------------------------------------------------------------
def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, ranked by (higher score, then lower index), returned in
    ascending index order.  -0.0 and +0.0 compare equal."""
    s = np.asarray(scores, np.float64)
    n = s.shape[0]
    if not (0 <= k <= n):
        raise ValueError("k out of range")
    if np.isnan(s).any():
        raise ValueError("NaN score")
    order = np.lexsort((np.arange(n), -s))      # primary: score descending; ties: index ascending
    return np.sort(order[:k]).astype(np.int64)


# ---------------------------------------------------------------------------------------------
# one attention layer over the kept tokens / heads of one sequence
# ---------------------------------------------------------------------------------------------
def attention_layer_seq(Q, K, V, heads, d_h: int, H: int, quant: bool, theta: float,
                        sm_scale: float, key_gain=None, flags_override=None, v_keep: int | None = None):
    """Q, K, V: [n, H*d_h] projections of the kept rows (all heads).  ``heads``: kept head ids.
    ``key_gain`` [n]: per-token factor applied to K after projection (boosted keys).  ``v_keep``:
    V vectors each head keeps under local value pruning (None: all); token importance uses the
    full probabilities, head importance the pruned outputs.

    Returns dict(O [n, H*d_h] with zeros for pruned heads, tok_inc [n], head_inc [H],
    flags {h: bool[n]}, pmax {h: [n]}, codes {h: (kq, vq)}, refetch (count of refetched rows)).
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    n = Q.shape[0]
    O = np.zeros((n, H * d_h))
    tok_inc = np.zeros(n)
    head_inc = np.zeros(H)
    flags, pmaxs, codes = {}, {}, {}
    refetch = 0
    for h in heads:
        sl = slice(h * d_h, (h + 1) * d_h)
        q, k, v = Q[:, sl], K[:, sl], V[:, sl]
        if quant:
            k32 = k.astype(np.float32)
            if key_gain is not None:
                k32 = k32 * np.asarray(key_gain, np.float32)[:, None]
            kq = quantize_head(k32)
            vq = quantize_head(v.astype(np.float32))
            fo = None if flags_override is None else flags_override.get(h)
            r = progressive_attention(q, kq, vq, theta, sm_scale, flags_override=fo, v_keep=v_keep)
            Oh, P = r["O"], r["P"]
            flags[h], pmaxs[h] = r["flags"], r["pmax_msb"]
            codes[h] = (kq, vq)
            refetch += int(r["flags"].sum())
        else:
            if key_gain is not None:
                k = k * np.asarray(key_gain, np.float64)[:, None]
            Oh, P, _ = dense_attention_value_pruned(q, k, v, sm_scale, v_keep)
        O[:, sl] = Oh
        tok_inc += token_importance_increment(P)
        head_inc[h] += head_importance_increment(Oh)
    return dict(O=O, tok_inc=tok_inc, head_inc=head_inc, flags=flags, pmax=pmaxs, codes=codes,
                refetch=refetch)


# ---------------------------------------------------------------------------------------------
# C6/C7  cascade prefill (summarization) over L layers (§II "Cascade pruning", §III.A)
# ---------------------------------------------------------------------------------------------
def cascade_prefill(X, w_qkv, w_o, H: int, d_h: int, token_keep, head_keep, quant: bool,
                    theta: float, sm_scale: float | None = None, key_gain=None):
    """Free-running cascade.  X [B,T,D]; w_qkv[l] [D, 3*H*d_h] = [W_q | W_k | W_v]; w_o[l]
    [H*d_h, D]; token_keep[l] = k_l tokens entering layer l (k_0 = T); head_keep[l] = H_l.

    Per layer l and sequence b: project the kept rows, run attention on the kept heads, add the
    column sums of P to the cumulative token importance I_b (original token ids) and sum|O_h| to
    the cumulative head importance J_b, update X_kept += O @ W_o; then (l < L-1) keep the top
    k_{l+1} tokens of S_l by I_b and the top H_{l+1} heads by J_b.  Pruned rows of X stay frozen.

    Returns dict(X (full [B,T,D], frozen rows kept), x_final [B, k_{L-1}, D], kept [L][B] arrays,
    heads [L][B] arrays, I [B,T], J [B,H], refetch [L], O [L][B] per-layer outputs, I_sel/J_sel
    [L-1] copies of I and J at each selection).
    """
    X = np.array(X, np.float64)
    B, T, D = X.shape
    L = len(w_qkv)
    HD = H * d_h
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d_h)
    I = np.zeros((B, T))
    J = np.zeros((B, H))
    kept = [np.arange(T) for _ in range(B)]
    heads = [np.arange(H) for _ in range(B)]
    kept_log, heads_log, O_log, refetch, I_sel, J_sel = [], [], [], [], [], []
    for l in range(L):
        assert all(len(s) == token_keep[l] for s in kept)
        assert all(len(hs) == head_keep[l] for hs in heads)
        kept_log.append([s.copy() for s in kept])
        heads_log.append([hs.copy() for hs in heads])
        O_l, rf = [], 0
        for b in range(B):
            S = kept[b]
            Xk = X[b, S]
            qkv = Xk @ w_qkv[l]
            gain = None if key_gain is None else np.asarray(key_gain)[b, S]
            r = attention_layer_seq(qkv[:, :HD], qkv[:, HD:2 * HD], qkv[:, 2 * HD:], heads[b],
                                    d_h, H, quant, theta, sm_scale, key_gain=gain)
            I[b, S] += r["tok_inc"]
            J[b] += r["head_inc"]
            X[b, S] = Xk + r["O"] @ w_o[l]
            O_l.append(r["O"])
            rf += r["refetch"]
        O_log.append(O_l)
        refetch.append(rf)
        if l < L - 1:
            I_sel.append(I.copy())
            J_sel.append(J.copy())
            for b in range(B):
                sel = topk_select(I[b, kept[b]], token_keep[l + 1])
                kept[b] = kept[b][sel]
                hsel = topk_select(J[b, heads[b]], head_keep[l + 1])
                heads[b] = heads[b][hsel]
    x_final = np.stack([X[b, kept[b]] for b in range(B)])
    return dict(X=X, x_final=x_final, kept=kept_log, heads=heads_log, I=I, J=J,
                refetch=refetch, O=O_log, I_sel=I_sel, J_sel=J_sel)


# ---------------------------------------------------------------------------------------------
# C8  decode (generation) step with cumulative importance (§II "Attention-based NLP models":
#     one new token per iteration against cached K and V)
# ---------------------------------------------------------------------------------------------
def decode_step(x, caches, n_old: int, I, w_qkv, w_o, H: int, d_h: int, keep_fn, theta: float,
                sm_scale: float | None = None, teacher: dict | None = None, v_keep_fn=None):
    """One generation step for B sequences.

    x [B, D]: this step's input rows.  caches[l]: dict with k_msb, k_lsb, v_msb, v_lsb
    ([B,H,cap,d_h], LSB unpacked), k_scale, v_scale ([B,H], prompt-time), mutated in place: the
    new token's K/V codes are appended at row n_old with the prompt-time scale (saturating).
    I [B, cap]: cumulative token importance, mutated in place.  keep_fn(n) -> [k_0..k_{L-1}].
    teacher (optional): {"qkv": [L] arrays [B, 3*H*d_h], "x": [L] arrays [B, D]} replaces the
    projections and layer inputs with given values (teacher forcing).  v_keep_fn (optional):
    v_keep_fn(l, k_l) -> V vectors each head of layer l keeps under local value pruning (its one
    query row's probabilities rank the keys); None keeps them all.

    Per layer l: q,k,v = x_l @ W; append k,v; attend over S_l (S_0 = all n rows); I += P;
    x_{l+1} = x_l + O @ W_o; S_{l+1} = top-k_{l+1}(I restricted to S_l).

    Returns dict(x_out [B,D], kept [L][B], O [L] [B, H*d_h], flags [L] [B,H], sat, xs [L+1]).
    """
    x = np.array(x, np.float64)
    B = x.shape[0]
    L = len(w_qkv)
    HD = H * d_h
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d_h)
    n = n_old + 1
    ks = keep_fn(n)
    kept = [np.arange(n) for _ in range(B)]
    kept_log, O_log, flag_log, xs = [], [], [], [x.copy()]
    sat = 0
    for l in range(L):
        if teacher is not None:
            x = np.array(teacher["x"][l], np.float64)
            qkv = np.array(teacher["qkv"][l], np.float64)
        else:
            qkv = x @ w_qkv[l]
        c = caches[l]
        kept_log.append([s.copy() for s in kept])
        O = np.zeros((B, HD))
        flags = np.zeros((B, H), bool)
        for b in range(B):
            S = kept[b]
            for h in range(H):
                sl = slice(h * d_h, (h + 1) * d_h)
                kq = quantize_head(qkv[b, HD + h * d_h: HD + (h + 1) * d_h][None].astype(np.float32),
                                   scale=c["k_scale"][b, h])
                vq = quantize_head(qkv[b, 2 * HD + h * d_h: 2 * HD + (h + 1) * d_h][None].astype(np.float32),
                                   scale=c["v_scale"][b, h])
                sat += kq["sat"] + vq["sat"]
                c["k_msb"][b, h, n_old] = kq["msb"][0]
                c["k_lsb"][b, h, n_old] = kq["lsb"][0]
                c["v_msb"][b, h, n_old] = vq["msb"][0]
                c["v_lsb"][b, h, n_old] = vq["lsb"][0]
                kblk = dict(msb=c["k_msb"][b, h, S], lsb=c["k_lsb"][b, h, S], scale=c["k_scale"][b, h])
                vblk = dict(msb=c["v_msb"][b, h, S], lsb=c["v_lsb"][b, h, S], scale=c["v_scale"][b, h])
                vk = None if v_keep_fn is None else v_keep_fn(l, len(S))
                r = progressive_attention(qkv[b, sl][None], kblk, vblk, theta, sm_scale, v_keep=vk)
                O[b, sl] = r["O"][0]
                flags[b, h] = r["flags"][0]
                I[b, S] += token_importance_increment(r["P"])
        x = x + O @ w_o[l]
        xs.append(x.copy())
        O_log.append(O)
        flag_log.append(flags)
        if l < L - 1:
            for b in range(B):
                sel = topk_select(I[b, kept[b]], ks[l + 1])
                kept[b] = kept[b][sel]
    return dict(x_out=x, kept=kept_log, O=O_log, flags=flag_log, sat=sat, xs=xs)


def empty_decode_caches(L: int, B: int, H: int, cap: int, d_h: int):
    """Zero-filled code planes (unpacked LSB) and unit scales for L layers."""
    return [dict(k_msb=np.zeros((B, H, cap, d_h), np.int8), k_lsb=np.zeros((B, H, cap, d_h), np.uint8),
                 v_msb=np.zeros((B, H, cap, d_h), np.int8), v_lsb=np.zeros((B, H, cap, d_h), np.uint8),
                 k_scale=np.ones((B, H), np.float32), v_scale=np.ones((B, H), np.float32))
            for _ in range(L)]


def quantize_prompt_cache(cache: dict, K32: np.ndarray, V32: np.ndarray):
    """Fill rows [0, T0) of one layer's cache from prompt K/V [B,H,T0,d_h] (float32), one
    amax scale per (sequence, head, tensor)."""
    B, H, T0, _ = K32.shape
    for b in range(B):
        for h in range(H):
            kq = quantize_head(K32[b, h])
            vq = quantize_head(V32[b, h])
            cache["k_msb"][b, h, :T0], cache["k_lsb"][b, h, :T0] = kq["msb"], kq["lsb"]
            cache["v_msb"][b, h, :T0], cache["v_lsb"][b, h, :T0] = vq["msb"], vq["lsb"]
            cache["k_scale"][b, h], cache["v_scale"][b, h] = kq["scale"], vq["scale"]
