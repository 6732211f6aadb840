"""GPU parity of spatten_attention_layer (all kernels) against the oracle.

Inputs: seeded draws cast to bf16/fp32 on the host.  K/V are quantized on the device (K1, whose
codes are checked bit-exact against the oracle's on the same values here too), so the oracle and
the kernel see identical 12-bit codes.  Criteria (from the workload's correctness statement):
max |O - O_ref| <= 2e-2 x RMS(O_ref) for bf16 queries, 1e-4 x RMS for the float32 path; token
importance within 2e-5 of the largest entry; refetch flags equal except at near-ties
(|1/ell - theta| <= 1e-5 theta), where the oracle is rerun with the kernel's decision.
"""
import math

import numpy as np
import pytest
import torch

from cascade_token_head_b200 import synth
from oracle import spatten_ref as R

from gpu_helpers import (BF, assert_close_bf16_out, assert_close_rms, host_cast, lib, oracle_quantize_blocks,
                         split_heads, to_dev, ws)

pytestmark = pytest.mark.gpu


def make_layer(B, H, n, d, seed, boost=0, dtype=BF, scale=1.0):
    g = synth.rng_for(seed)
    raw = g.standard_normal((B, n, 3 * H * d)) * scale
    gain = np.ones((B, n), np.float32)
    if boost:
        for b in range(B):
            gain[b, g.choice(n, boost, replace=False)] = 4.0
    return raw, gain


def run_layer(S, raw, gain, B, H, n, d, theta, heads=None, kernel=0, dtype=BF, kv_idx=None, n_q=None,
              cap=None, quantized=True, v_keep=0):
    """Quantize K/V on the device and run the attention layer.  Returns dict of host arrays."""
    esz = 2 if dtype == BF else 4
    x = to_dev(raw, dtype)
    HD = H * d
    cap = cap or n
    n_q = n_q or n
    msbk = torch.zeros((B, H, cap, d), dtype=torch.int8, device="cuda")
    lsbk = torch.zeros((B, H, cap, d // 2), dtype=torch.uint8, device="cuda")
    msbv, lsbv = torch.zeros_like(msbk), torch.zeros_like(lsbk)
    sk = torch.zeros(B * H, dtype=torch.float32, device="cuda")
    sv = torch.zeros_like(sk)
    a = S.attn_args()
    a.B, a.H, a.n_q, a.d_h = B, H, n_q, d
    if quantized:
        S.quantize_kv(x.data_ptr() + HD * esz, B, H, cap, d, 3 * HD, msbk, lsbk, cap, 0, scale_out=sk,
                      row_gain=to_dev(gain), ld_gain=cap, dtype=S.dtype_code(x))
        S.quantize_kv(x.data_ptr() + 2 * HD * esz, B, H, cap, d, 3 * HD, msbv, lsbv, cap, 0, scale_out=sv,
                      dtype=S.dtype_code(x))
        a.quantized = 1
        a.k_msb, a.k_lsb, a.k_scale = msbk.data_ptr(), lsbk.data_ptr(), sk.data_ptr()
        a.v_msb, a.v_lsb, a.v_scale = msbv.data_ptr(), lsbv.data_ptr(), sv.data_ptr()
        a.kv_cap = cap
    else:
        a.quantized = 0
        a.k, a.v = x.data_ptr() + HD * esz, x.data_ptr() + 2 * HD * esz
        a.kv_dtype, a.kv_ld_tok = S.dtype_code(x), 3 * HD
    n_kv = n if kv_idx is None else kv_idx.shape[1]
    a.n_kv = n_kv
    if kv_idx is not None:
        kvi = to_dev(kv_idx, torch.int32)
        a.kv_idx, a.kv_idx_ld = kvi.data_ptr(), kv_idx.shape[1]
    hk = heads.shape[1] if heads is not None else H
    a.H_kept = hk
    if heads is not None:
        hd = to_dev(heads, torch.int32)
        a.head_idx, a.head_idx_ld = hd.data_ptr(), hk
    xq = x if n_q == x.shape[1] else x[:, :n_q, :].contiguous()   # batch stride of q is n_q rows
    a.q, a.q_dtype, a.q_ld_tok = xq.data_ptr(), S.dtype_code(x), 3 * HD
    o = torch.full((B, n_q, HD), 7.0, dtype=dtype, device="cuda")
    a.o, a.o_ld_tok, a.zero_pruned_heads = o.data_ptr(), HD, 1
    cap_t = max(cap, n_kv)
    tok = torch.zeros((B, cap_t), dtype=torch.float32, device="cuda")
    hed = torch.zeros((B, H), dtype=torch.float32, device="cuda")
    flags = torch.full((B, H, n_q), 9, dtype=torch.uint8, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    a.tok_imp, a.tok_imp_ld = tok.data_ptr(), cap_t
    if kv_idx is not None:
        a.tok_imp_map, a.tok_imp_map_ld = kvi.data_ptr(), kv_idx.shape[1]
    a.head_imp, a.refetch_flags, a.refetch_count = hed.data_ptr(), flags.data_ptr(), cnt.data_ptr()
    a.refetch_threshold, a.kernel, a.v_keep = theta, kernel, v_keep
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    a.dev_status = st.data_ptr()
    w = ws(S.attention_workspace_size(a))
    S.attention_layer(a, w, w.numel())
    torch.cuda.synchronize()
    out = dict(o=o.float().cpu().numpy(), tok=tok.cpu().numpy(), head=hed.cpu().numpy(),
               flags=flags.cpu().numpy(), count=int(cnt.item()), status=int(st.item()))
    if quantized:
        out.update(msbk=msbk.cpu().numpy(), lsbk=lsbk.cpu().numpy(), sk=sk.cpu().numpy().reshape(B, H),
                   msbv=msbv.cpu().numpy(), lsbv=lsbv.cpu().numpy(), sv=sv.cpu().numpy().reshape(B, H))
    return out


def oracle_layer(raw, gain, B, H, n, d, theta, heads, dtype, got, kv_idx=None, n_q=None, quantized=True,
                 v_keep=None):
    """Oracle over the same host-cast values; returns O, token/head importance, flags, pmax (and,
    with v_keep, each head's kept V set and its column sums)."""
    vals = host_cast(raw, dtype)
    Q = split_heads(vals, H, d, 0)
    K = split_heads(vals, H, d, 1).astype(np.float32)
    V = split_heads(vals, H, d, 2).astype(np.float32)
    n_q = n_q or n
    sm = 1.0 / math.sqrt(d)
    if quantized:
        mk, lk, sk = oracle_quantize_blocks(K, gain)
        mv, lv, sv = oracle_quantize_blocks(V)
        np.testing.assert_array_equal(got["msbk"], mk)
        np.testing.assert_array_equal(got["lsbk"], lk)
        np.testing.assert_array_equal(got["msbv"], mv)
        np.testing.assert_array_equal(got["sk"], sk)
    n_kv_cols = got["tok"].shape[1]
    O = np.zeros((B, n_q, H * d))
    tok = np.zeros((B, n_kv_cols))
    head = np.zeros((B, H))
    flags = np.zeros((B, H, n_q), bool)
    kept, colsum = {}, {}
    near = 0
    for b in range(B):
        hs = range(H) if heads is None else heads[b]
        rows = np.arange(n) if kv_idx is None else kv_idx[b]
        for h in hs:
            q = Q[b, h, :n_q]
            if quantized:
                kq = dict(msb=mk[b, h, rows], lsb=R.unpack_lsb(lk[b, h, rows]), scale=sk[b, h])
                vq = dict(msb=mv[b, h, rows], lsb=R.unpack_lsb(lv[b, h, rows]), scale=sv[b, h])
                r = R.progressive_attention(q, kq, vq, theta, sm, v_keep=v_keep)
                gf = got["flags"][b, h].astype(bool)
                diff = gf != r["flags"]
                if diff.any():
                    # only near-ties may disagree; then follow the kernel's decision
                    assert np.all(np.abs(r["pmax_msb"][diff] - theta) <= 1e-5 * theta), "flag mismatch off a tie"
                    near += int(diff.sum())
                    r = R.progressive_attention(q, kq, vq, theta, sm, flags_override=gf, v_keep=v_keep)
                Oh, P = r["O"], r["P"]
                flags[b, h] = r["flags"]
                kept[b, h] = r["v_kept"]
            else:
                Oh, P, kept[b, h] = R.dense_attention_value_pruned(q, K[b, h][rows], V[b, h][rows], sm, v_keep)
            colsum[b, h] = P.sum(axis=0)
            O[b, :, h * d:(h + 1) * d] = Oh
            tok[b, rows] += R.token_importance_increment(P)
            head[b, h] += R.head_importance_increment(Oh)
    return dict(O=O, tok=tok, head=head, flags=flags, near=near, kept=kept, colsum=colsum)


def check(got, ref, heads, H, d, tol_o, tol_head, dtype_name):
    B = got["o"].shape[0]
    kept_cols = [np.concatenate([np.arange(h * d, (h + 1) * d) for h in (range(H) if heads is None else heads[b])])
                 for b in range(B)]
    go = np.stack([got["o"][b][:, kept_cols[b]] for b in range(B)])
    ro = np.stack([ref["O"][b][:, kept_cols[b]] for b in range(B)])
    if dtype_name == "fp32":
        assert_close_rms(go, ro, tol_o, "O (fp32)")
    else:
        assert_close_bf16_out(go, ro, tol_o, f"O ({dtype_name})")
    # pruned heads are zero-filled
    if heads is not None:
        for b in range(B):
            for h in range(H):
                if h not in heads[b]:
                    assert np.all(got["o"][b, :, h * d:(h + 1) * d] == 0)
    np.testing.assert_allclose(got["tok"], ref["tok"], rtol=0, atol=2e-5 * np.abs(ref["tok"]).max())
    np.testing.assert_allclose(got["head"], ref["head"], rtol=tol_head, atol=1e-6)
    for b in range(B):
        for h in (range(H) if heads is None else heads[b]):
            np.testing.assert_array_equal(got["flags"][b, h].astype(bool), ref["flags"][b, h])
    assert got["count"] == int(ref["flags"].sum())


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("B,H,n,d,theta,boost,keep", [
    (2, 4, 64, 64, 0.1, 3, None), (2, 4, 200, 64, 0.1, 10, [0, 2, 3]), (1, 2, 333, 128, 0.1, 12, None),
    (2, 3, 129, 64, 0.0, 0, None), (2, 3, 129, 64, 2.0, 0, [1]), (3, 12, 512, 64, 0.1, 26, list(range(0, 12, 2)))])
def test_attention_quantized_bf16(cuda, kernel, B, H, n, d, theta, boost, keep):
    S = lib()
    raw, gain = make_layer(B, H, n, d, seed=n * 31 + d + B, boost=boost)
    heads = None if keep is None else np.array([keep] * B, np.int32)
    got = run_layer(S, raw, gain, B, H, n, d, theta, heads=heads, kernel=kernel)
    ref = oracle_layer(raw, gain, B, H, n, d, theta, heads, BF, got)
    check(got, ref, heads, H, d, 2e-2, 1e-2, "bf16")


@pytest.mark.parametrize("n", [1, 7, 128, 200])
def test_attention_fp32_unquantized(cuda, n):
    """The float32 configuration's layer: no quantization, fp32 everywhere."""
    S = lib()
    B, H, d = 1, 4, 64
    raw, gain = make_layer(B, H, n, d, seed=n)
    got = run_layer(S, raw, None, B, H, n, d, 0.0, dtype=torch.float32, quantized=False)
    ref = oracle_layer(raw, None, B, H, n, d, 0.0, None, torch.float32, got, quantized=False)
    check(got, ref, None, H, d, 1e-4, 1e-5, "fp32")


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("d,theta,cap,n_kv,keep", [
    (64, 0.2, 300, 211, None), (64, 0.0, 300, 211, None), (128, 0.2, 300, 211, None),
    (64, 0.2, 40, 7, None), (64, 0.2, 2600, 2048, None), (128, 0.05, 2600, 2047, [1, 3]),
    (64, 0.2, 3000, 2500, None), (128, 0.2, 1300, 1153, [0, 2, 3])])
def test_attention_decode_index_listed(cuda, kernel, d, theta, cap, n_kv, keep):
    """One query row per (sequence, head) against an index-listed subset of a cache, through the
    decode path (the items kernel over runs of the listed keys, then the per-sequence combine) and,
    with kernel=1, through the float32 CUDA-core kernel on the same inputs.  Lists from 7 to 2500
    keys, ragged last items, pruned heads."""
    S = lib()
    B, H = 3, 4
    g = synth.rng_for(d + int(theta * 10) + n_kv)
    raw, gain = make_layer(B, H, cap, d, seed=99 + d)
    kv_idx = np.stack([np.sort(g.choice(cap, n_kv, replace=False)) for _ in range(B)]).astype(np.int32)
    heads = None if keep is None else np.array([keep] * B, np.int32)
    got = run_layer(S, raw, gain, B, H, cap, d, theta, heads=heads, kernel=kernel, kv_idx=kv_idx, n_q=1)
    ref = oracle_layer(raw, gain, B, H, cap, d, theta, heads, BF, got, kv_idx=kv_idx, n_q=1)
    check(got, ref, heads, H, d, 2e-2, 1e-2, "decode")
    # importance lands only on the listed rows
    for b in range(B):
        mask = np.ones(cap, bool)
        mask[kv_idx[b]] = False
        assert np.all(got["tok"][b, mask] == 0)


@pytest.mark.parametrize("d,cap,n_kv,keep", [(64, 1300, 1153, None), (128, 700, 611, [0, 2, 3]), (64, 300, 7, None)])
def test_decode_predicated_lsb_fetch(cuda, d, cap, n_kv, keep):
    """SPATTEN_ATTN_DECODE_PREDICATED: the MSB planes of every row, the refetch decision, then the
    LSB planes of the flagged rows only.  With a threshold at which some rows refetch and others
    do not, its outputs, importances, flags and count are bit-identical to the single-pass decode
    kernel's (SPATTEN_ATTN_DECODE), and they match the oracle; at theta 0 it is the MSB pass."""
    S = lib()
    B, H = 4, 4
    g = synth.rng_for(7 * d + n_kv)
    raw, gain = make_layer(B, H, cap, d, seed=41 + d, boost=max(1, cap // 12))
    kv_idx = np.stack([np.sort(g.choice(cap, n_kv, replace=False)) for _ in range(B)]).astype(np.int32)
    heads = None if keep is None else np.array([keep] * B, np.int32)
    rows = B * (H if keep is None else len(keep))
    # a threshold between the rows' MSB-pass maximum probabilities: some rows refetch, some not
    theta, single = None, None
    for t in (0.5, 0.3, 0.2, 0.1, 0.05, 0.02, 0.01, 0.005, 0.002):
        single = run_layer(S, raw, gain, B, H, cap, d, t, heads=heads, kernel=S.ATTN_DECODE, kv_idx=kv_idx, n_q=1)
        if 0 < single["count"] < rows:
            theta = t
            break
    assert theta is not None, "no threshold splits the rows"
    pred = run_layer(S, raw, gain, B, H, cap, d, theta, heads=heads, kernel=S.ATTN_DECODE_PREDICATED,
                     kv_idx=kv_idx, n_q=1)
    print(f"theta {theta}: {single['count']} of {rows} rows refetch")
    for key in ("o", "tok", "head", "flags", "count", "status"):
        np.testing.assert_array_equal(pred[key], single[key])
    ref = oracle_layer(raw, gain, B, H, cap, d, theta, heads, BF, pred, kv_idx=kv_idx, n_q=1)
    check(pred, ref, heads, H, d, 2e-2, 1e-2, "decode (predicated)")
    zero = run_layer(S, raw, gain, B, H, cap, d, 0.0, heads=heads, kernel=S.ATTN_DECODE_PREDICATED, kv_idx=kv_idx,
                     n_q=1)
    zero_single = run_layer(S, raw, gain, B, H, cap, d, 0.0, heads=heads, kernel=S.ATTN_DECODE, kv_idx=kv_idx, n_q=1)
    for key in ("o", "tok", "head", "count"):
        np.testing.assert_array_equal(zero[key], zero_single[key])


def test_attention_deterministic(cuda):
    S = lib()
    B, H, n, d = 2, 6, 300, 64
    raw, gain = make_layer(B, H, n, d, seed=5, boost=15)
    a = run_layer(S, raw, gain, B, H, n, d, 0.1)
    b = run_layer(S, raw, gain, B, H, n, d, 0.1)
    np.testing.assert_array_equal(a["tok"], b["tok"])
    np.testing.assert_array_equal(a["head"], b["head"])
    np.testing.assert_array_equal(a["o"], b["o"])


def test_attention_query_out_of_fp16_range_reports_status(cuda):
    """The tensor-core kernels take fp16 operands: a bf16 query value past fp16's range is stored
    saturated, and the call reports SPATTEN_E_RANGE in dev_status (in-range calls report 0)."""
    S = lib()
    B, H, n, d = 1, 2, 130, 64
    for big, want in ((3.0, S.OK), (1.0e5, S.E_RANGE)):
        raw, gain = make_layer(B, H, n, d, seed=31)
        raw[0, 77, 5] = big                       # one element of head 0's query row 77
        x = to_dev(raw, BF)
        HD = H * d
        planes = []
        for t in (1, 2):
            msb = torch.zeros((B, H, n, d), dtype=torch.int8, device="cuda")
            lsb = torch.zeros((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
            sc = torch.zeros(B * H, device="cuda")
            S.quantize_kv(x.data_ptr() + t * HD * 2, B, H, n, d, 3 * HD, msb, lsb, n, 0, scale_out=sc, dtype=S.BF16)
            planes.append((msb, lsb, sc))
        a = S.attn_args()
        a.B, a.H, a.n_q, a.n_kv, a.d_h, a.H_kept = B, H, n, n, d, H
        a.q, a.q_dtype, a.q_ld_tok = x.data_ptr(), S.BF16, 3 * HD
        a.quantized, a.kv_cap = 1, n
        a.k_msb, a.k_lsb, a.k_scale = (t.data_ptr() for t in planes[0])
        a.v_msb, a.v_lsb, a.v_scale = (t.data_ptr() for t in planes[1])
        o = torch.zeros((B, n, HD), dtype=BF, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        a.o, a.o_ld_tok, a.dev_status, a.refetch_threshold = o.data_ptr(), HD, st.data_ptr(), 0.1
        a.kernel = S.ATTN_TENSOR_CORE
        w = ws(S.attention_workspace_size(a))
        S.attention_layer(a, w, w.numel())
        torch.cuda.synchronize()
        assert int(st.item()) == want


def test_forced_timeout_reports_status_and_context_survives(cuda):
    """The tensor-core kernels' bounded waits run out on purpose (spatten_set_wait_limit(1): one
    poll per pipeline wait): the call reports SPATTEN_E_TIMEOUT in its status word and its kernels
    return (the synchronize inside run_layer ends); the context stays usable: with the default
    limit restored the same call reports 0 and repeats, bit for bit, the results of a run made
    before the forced timeout."""
    S = lib()
    B, H, n, d = 1, 2, 130, 64
    raw, gain = make_layer(B, H, n, d, seed=31, boost=5)
    before = run_layer(S, raw, gain, B, H, n, d, 0.1, kernel=S.ATTN_TENSOR_CORE)
    assert before["status"] == S.OK
    try:
        S.set_wait_limit(1)
        timed_out = run_layer(S, raw, gain, B, H, n, d, 0.1, kernel=S.ATTN_TENSOR_CORE)
    finally:
        S.set_wait_limit(0)
    assert timed_out["status"] == S.E_TIMEOUT
    after = run_layer(S, raw, gain, B, H, n, d, 0.1, kernel=S.ATTN_TENSOR_CORE)
    assert after["status"] == S.OK
    for key in ("o", "tok", "head", "flags", "count"):
        np.testing.assert_array_equal(after[key], before[key])
