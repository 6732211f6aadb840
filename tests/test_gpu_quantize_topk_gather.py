"""GPU parity of K1 (quantize), K4 (top-k) and K5 (gather) against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

from cascade_token_head_b200 import synth
from oracle import spatten_ref as R

from gpu_helpers import BF, host_cast, lib, oracle_quantize_blocks, split_heads, to_dev

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------------------------
# K1 quantize
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,B,H,n,d,gain", [
    (BF, 2, 3, 1, 64, False), (BF, 2, 3, 7, 64, True), (BF, 3, 4, 517, 64, True), (BF, 1, 2, 300, 128, False),
    (torch.float32, 2, 2, 129, 64, False), (BF, 1, 2, 5000, 128, True)])
def test_quantize_bit_exact(cuda, dtype, B, H, n, d, gain):
    S = lib()
    g = synth.rng_for(n * 7 + d)
    raw = g.standard_normal((B, n, 3 * H * d)) * 3.0
    x = to_dev(raw, dtype)
    gains = None
    if gain:
        gains = np.ones((B, n), np.float32)
        gains[:, g.choice(n, size=max(1, n // 20), replace=False)] = 4.0
    esz = 2 if dtype == BF else 4
    msb = torch.zeros((B, H, n, d), dtype=torch.int8, device="cuda")
    lsb = torch.zeros((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(B * H, dtype=torch.float32, device="cuda")
    gdev = to_dev(gains) if gain else None
    S.quantize_kv(x.data_ptr() + H * d * esz, B, H, n, d, 3 * H * d, msb, lsb, n, 0, scale_out=sc,
                  row_gain=gdev, ld_gain=n, dtype=S.dtype_code(x))
    torch.cuda.synchronize()
    k32 = split_heads(host_cast(raw, dtype), H, d, 1).astype(np.float32)
    m_ref, l_ref, s_ref = oracle_quantize_blocks(k32, gains)
    np.testing.assert_array_equal(sc.cpu().numpy().reshape(B, H), s_ref)
    np.testing.assert_array_equal(msb.cpu().numpy(), m_ref)
    np.testing.assert_array_equal(lsb.cpu().numpy(), l_ref)


def _half_boundary_values(s, count, rng):
    """float32 values at and a few ulps around (k + 1/2) s for integer k across the code range,
    plus the float32 neighbours of the exact quotient boundaries."""
    k = rng.integers(-2047, 2047, size=count)
    centre = ((k + 0.5) * np.float64(s)).astype(np.float32)
    steps = rng.integers(-3, 4, size=count)
    out = centre.copy()
    for i, st in enumerate(steps):
        v = centre[i]
        for _ in range(abs(int(st))):
            v = np.nextafter(v, np.float32(np.inf) if st > 0 else np.float32(-np.inf))
        out[i] = v
    return out


@pytest.mark.parametrize("s", [0.0013672, 0.1, 1.0 / 3.0, 7.123e-5])
def test_quantize_half_integer_boundaries_fixed_scale(cuda, s):
    """Codes of values crafted at rounding boundaries of x/s (the fast reciprocal path must defer
    to the IEEE quotient there): bit-exact against the oracle's float32 division."""
    S = lib()
    rng = synth.rng_for(int(s * 1e7) % 10007)
    B, H, n, d, cap = 2, 2, 64, 64, 64
    s32 = np.float32(s)
    vals = _half_boundary_values(s32, B * n * H * d, rng).reshape(B, n, H * d)
    x = to_dev(vals, torch.float32)
    msb = torch.zeros((B, H, cap, d), dtype=torch.int8, device="cuda")
    lsb = torch.zeros((B, H, cap, d // 2), dtype=torch.uint8, device="cuda")
    sat = torch.zeros(1, dtype=torch.int32, device="cuda")
    scales = to_dev(np.full(B * H, s32, np.float32))
    S.quantize_kv(x, B, H, n, d, H * d, msb, lsb, cap, 0, scale_in=scales, sat_count=sat, dtype=S.F32)
    torch.cuda.synchronize()
    x32 = vals.reshape(B, n, H, d).transpose(0, 2, 1, 3)
    want_sat = 0
    for b in range(B):
        for h in range(H):
            r = R.quantize_head(np.ascontiguousarray(x32[b, h]), scale=s32)
            want_sat += r["sat"]
            np.testing.assert_array_equal(msb[b, h].cpu().numpy(), r["msb"])
            np.testing.assert_array_equal(lsb[b, h].cpu().numpy(), R.pack_lsb(r["lsb"]))
    assert int(sat.item()) == want_sat


def test_quantize_half_integer_boundaries_amax_scale(cuda):
    """The same with the scale derived from the block's amax on the device."""
    S = lib()
    rng = synth.rng_for(4242)
    B, H, n, d = 2, 3, 256, 64
    vals = np.empty((B, n, H * d), np.float32)
    for b in range(B):
        for h in range(H):
            amax = np.float32(rng.uniform(0.5, 9.0))
            s = np.float32(amax / np.float32(2047.0))
            blk = _half_boundary_values(s, n * d, rng).reshape(n, d)
            blk = np.clip(blk, -amax, amax)
            blk[0, 0] = amax
            vals[b, :, h * d:(h + 1) * d] = blk
    x = to_dev(vals, torch.float32)
    msb = torch.zeros((B, H, n, d), dtype=torch.int8, device="cuda")
    lsb = torch.zeros((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(B * H, dtype=torch.float32, device="cuda")
    S.quantize_kv(x, B, H, n, d, H * d, msb, lsb, n, 0, scale_out=sc, dtype=S.F32)
    torch.cuda.synchronize()
    m_ref, l_ref, s_ref = oracle_quantize_blocks(np.ascontiguousarray(vals.reshape(B, n, H, d).transpose(0, 2, 1, 3)))
    np.testing.assert_array_equal(sc.cpu().numpy().reshape(B, H), s_ref)
    np.testing.assert_array_equal(msb.cpu().numpy(), m_ref)
    np.testing.assert_array_equal(lsb.cpu().numpy(), l_ref)


@pytest.mark.parametrize("gain", [False, True])
def test_quantize_half_integer_boundaries_amax_scale_bf16(cuda, gain):
    """bf16 blocks (the paired-arithmetic path of the amax kernel): values rounded to bf16 at and
    one or two bf16 steps around (k + 1/2) s for small |k| (where bf16 steps are finer than one
    code), with and without a row gain; bit-exact against the oracle."""
    S = lib()
    rng = synth.rng_for(4343 + gain)
    B, H, n, d = 2, 3, 256, 64
    vals = np.empty((B, n, H * d), np.float32)
    for b in range(B):
        for h in range(H):
            amax = np.float32(torch.tensor(rng.uniform(0.5, 9.0)).to(BF).float().item())
            s = np.float32(amax / np.float32(2047.0))
            k = rng.integers(-120, 120, size=n * d)
            centre = torch.from_numpy(((k + 0.5) * np.float64(s)).astype(np.float32)).to(BF)
            bits = centre.view(torch.int16).to(torch.int32) + torch.from_numpy(rng.integers(-2, 3, size=n * d)).to(torch.int32)
            blk = bits.to(torch.int16).view(BF).float().numpy().reshape(n, d)
            blk = np.clip(blk, -amax, amax)
            blk[0, 0] = amax
            vals[b, :, h * d:(h + 1) * d] = blk
    gains = None
    if gain:
        gains = np.ones((B, n), np.float32)
        gains[:, rng.choice(n, size=12, replace=False)] = 4.0
    x = to_dev(vals, BF)
    assert np.array_equal(x.float().cpu().numpy(), vals)   # every value is a bf16
    msb = torch.zeros((B, H, n, d), dtype=torch.int8, device="cuda")
    lsb = torch.zeros((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
    sc = torch.zeros(B * H, dtype=torch.float32, device="cuda")
    S.quantize_kv(x, B, H, n, d, H * d, msb, lsb, n, 0, scale_out=sc, row_gain=to_dev(gains) if gain else None,
                  ld_gain=n, dtype=S.BF16)
    torch.cuda.synchronize()
    m_ref, l_ref, s_ref = oracle_quantize_blocks(np.ascontiguousarray(vals.reshape(B, n, H, d).transpose(0, 2, 1, 3)),
                                                 gains)
    np.testing.assert_array_equal(sc.cpu().numpy().reshape(B, H), s_ref)
    np.testing.assert_array_equal(msb.cpu().numpy(), m_ref)
    np.testing.assert_array_equal(lsb.cpu().numpy(), l_ref)


def test_quantize_full_size_bert_layer0(cuda):
    """K of the BERT-base layer-0 projection shape [32, 12, 512, 64], bf16, with boosted rows."""
    S = lib()
    w = synth.bert_base_prefill()
    g = synth.rng_for(1)
    B, H, n, d = w.B, w.H, w.T, w.d_h
    raw = g.standard_normal((B, n, 3 * H * d))
    x = to_dev(raw, BF)
    gains = np.ones((B, n), np.float32)
    for b in range(B):
        gains[b, g.choice(n, 26, replace=False)] = 4.0
    msb = torch.empty((B, H, n, d), dtype=torch.int8, device="cuda")
    lsb = torch.empty((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
    sc = torch.empty(B * H, dtype=torch.float32, device="cuda")
    S.quantize_kv(x.data_ptr() + H * d * 2, B, H, n, d, 3 * H * d, msb, lsb, n, 0, scale_out=sc,
                  row_gain=to_dev(gains), ld_gain=n, dtype=S.BF16)
    torch.cuda.synchronize()
    k32 = split_heads(host_cast(raw, BF), H, d, 1).astype(np.float32)
    m_ref, l_ref, s_ref = oracle_quantize_blocks(k32, gains)
    np.testing.assert_array_equal(sc.cpu().numpy().reshape(B, H), s_ref)
    np.testing.assert_array_equal(msb.cpu().numpy(), m_ref)
    np.testing.assert_array_equal(lsb.cpu().numpy(), l_ref)


def test_quantize_append_with_scale_saturates(cuda):
    S = lib()
    B, H, d, cap = 2, 3, 64, 10
    g = synth.rng_for(5)
    raw = g.standard_normal((B, 1, 3 * H * d)) * 2.0
    x = to_dev(raw, BF)
    scales = np.full(B * H, 0.001, np.float32)      # small scale: many codes saturate
    scales[0] = 0.05
    msb = torch.zeros((B, H, cap, d), dtype=torch.int8, device="cuda")
    lsb = torch.zeros((B, H, cap, d // 2), dtype=torch.uint8, device="cuda")
    sat = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.quantize_kv(x.data_ptr() + 2 * H * d * 2, B, H, 1, d, 3 * H * d, msb, lsb, cap, 7, scale_in=to_dev(scales),
                  sat_count=sat, dtype=S.BF16)
    torch.cuda.synchronize()
    v32 = split_heads(host_cast(raw, BF), H, d, 2).astype(np.float32)
    want_sat = 0
    for b in range(B):
        for h in range(H):
            r = R.quantize_head(v32[b, h], scale=scales[b * H + h])
            want_sat += r["sat"]
            np.testing.assert_array_equal(msb[b, h, 7].cpu().numpy(), r["msb"][0])
            np.testing.assert_array_equal(lsb[b, h, 7].cpu().numpy(), R.pack_lsb(r["lsb"])[0])
    assert int(sat.item()) == want_sat > 0
    assert int(msb[:, :, :7].abs().sum().item()) == 0 and int(msb[:, :, 8:].abs().sum().item()) == 0


# ------------------------------------------------------------------------------------------------
# K4 top-k
# ------------------------------------------------------------------------------------------------
def _topk_gpu(S, scores_np, k, map_np=None, with_ws=True):
    """with_ws: pass the optional workspace (spatten_topk_workspace_size), which lets long direct
    rows take the streaming path."""
    R_, n = scores_np.shape if map_np is None else map_np.shape
    sc = to_dev(scores_np)
    out = torch.full((R_, max(k, 1)), -1, dtype=torch.int32, device="cuda")
    comp = torch.full((R_, max(k, 1)), -1, dtype=torch.int32, device="cuda") if map_np is not None else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    mp = to_dev(map_np, torch.int32) if map_np is not None else None
    nb = S.topk_workspace_size(R_, n, k) if with_ws else 0
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    S.topk_select(sc, R_, n, scores_np.shape[1], k, out, max(k, 1), map=mp, ld_map=n if mp is not None else 0,
                  comp_out=comp, ws=ws, ws_bytes=nb, dev_status=st)
    torch.cuda.synchronize()
    return out.cpu().numpy()[:, :k], (comp.cpu().numpy()[:, :k] if comp is not None else None), int(st.item())


@pytest.mark.parametrize("R_,n,k,kind", [
    (3, 1, 1, "u"), (3, 1, 0, "u"), (4, 10, 3, "ties"), (5, 100, 100, "u"), (5, 100, 1, "u"),
    (8, 517, 200, "ties"), (4, 4097, 2048, "zeros"), (6, 20000, 13, "ln"), (2, 70000, 35000, "ties"),
    (3, 1000, 500, "const"),
    # row-length boundaries of the short-row kernels (warp per row <= 512, 4 warps <= 2048,
    # 16 warps <= 8192, clusters beyond), odd row counts, mixed signs, k = 1 and k = n - 1
    (7, 512, 461, "neg"), (5, 513, 1, "neg"), (6, 2048, 2047, "ties"), (3, 2049, 1024, "neg"),
    (2, 8192, 4096, "u"), (2, 8193, 819, "neg"), (9, 12, 11, "neg"), (1, 1153, 1131, "const"),
    (13, 160, 144, "ties")])
def test_topk_matches_oracle(cuda, R_, n, k, kind):
    S = lib()
    g = synth.rng_for(n + k)
    if kind == "u":
        x = g.random((R_, n)).astype(np.float32)
    elif kind == "ln":
        x = g.lognormal(0, 2, (R_, n)).astype(np.float32)
    elif kind == "ties":
        x = (g.integers(0, 5, (R_, n)) * 0.25 - 0.5).astype(np.float32)
    elif kind == "neg":
        x = g.standard_normal((R_, n)).astype(np.float32)
        x[:, ::11] = x[:, 3:4]   # exact duplicates across the sign boundary
    elif kind == "zeros":
        x = np.where(g.random((R_, n)) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
        x[:, ::7] = -1.0
    else:
        x = np.full((R_, n), 3.0, np.float32)
    got, _, st = _topk_gpu(S, x, k)
    assert st == 0
    for r in range(R_):
        np.testing.assert_array_equal(got[r], R.topk_select(x[r].astype(np.float64), k))


def test_topk_through_map_with_composition(cuda):
    S = lib()
    g = synth.rng_for(11)
    Rr, T, n, k = 4, 900, 600, 250
    imp = g.random((Rr, T)).astype(np.float32)
    imp[:, ::10] = imp[:, 1::10]                    # ties across the gathered list
    mp = np.stack([np.sort(g.choice(T, n, replace=False)) for _ in range(Rr)]).astype(np.int32)
    got, comp, st = _topk_gpu(S, imp, k, mp)
    assert st == 0
    for r in range(Rr):
        sel = R.topk_select(imp[r, mp[r]].astype(np.float64), k)
        np.testing.assert_array_equal(got[r], sel)
        np.testing.assert_array_equal(comp[r], mp[r][sel])


@pytest.mark.parametrize("n,k,pos", [(50, 10, 7), (70001, 7000, 123), (70001, 7000, 69999), (70001, 63000, 5)])
def test_topk_nan_reports_status(cuda, n, k, pos):
    """A NaN anywhere in a row gives E_NONFINITE: short rows, and long rows on the streaming path
    (the NaN passes the filter's window tests and is seen among the candidates)."""
    S = lib()
    x = synth.rng_for(n + pos).random((2, n)).astype(np.float32)
    x[1, pos] = np.nan
    _, _, st = _topk_gpu(S, x, k)
    assert st == S.E_NONFINITE


@pytest.mark.parametrize("N", [1024, 16384, 262144, 1048576])
@pytest.mark.parametrize("dist", ["uniform", "lognormal"])
def test_topk_sweep_full_size(cuda, N, dist):
    """The top-k sweep workload (64 rows, 1 % exact duplicates), k = 10 % and 50 % of N.
    Every row is checked bit-exact against the oracle (which also fixes which members of a tie
    group at the threshold are taken: the lowest indices), plus the selection properties."""
    S = lib()
    x = synth.draw_topk_row_block(64, N, dist, 0.01, seed=N % 9973 + (dist == "lognormal"))
    rows = range(64)
    for frac in (0.1, 0.5):
        k = int(frac * N)
        got, _, st = _topk_gpu(S, x, k)
        assert st == 0
        for r in rows:
            np.testing.assert_array_equal(got[r], R.topk_select(x[r].astype(np.float64), k))
        # properties on every row: ascending, k distinct, threshold rule with lower-index ties
        assert np.all(np.diff(got, axis=1) > 0)
        for r in range(64):
            kth = np.partition(x[r], N - k)[N - k]
            sel_vals = x[r][got[r]]
            assert np.all(sel_vals >= kth) and np.count_nonzero(x[r] > kth) <= k


@pytest.mark.parametrize("with_ws", [True, False])
def test_topk_long_rows_bracket_misses_fall_back(cuda, with_ws):
    """Long rows on the streaming path (with the workspace) where the sample bracket cannot hold the
    k-th key -- all-equal rows, five distinct values, a row sorted by index -- are redone by the
    cluster kernel; ordinary rows in the same call stay on the streaming path.  Without the
    workspace every row takes the cluster kernel.  All rows bit-exact."""
    S = lib()
    g = synth.rng_for(77)
    R_, n = 6, 70001
    x = g.random((R_, n)).astype(np.float32)
    x[1] = 2.5                                                     # all equal
    x[3] = (g.integers(0, 5, n) * 0.5).astype(np.float32)         # five distinct values
    x[4] = np.linspace(-1.0, 1.0, n, dtype=np.float32)            # sorted by index
    x[5, ::3] = -x[5, ::3]                                         # mixed signs
    for k in (1, 7000, 35000, n - 1):
        got, _, st = _topk_gpu(S, x, k, with_ws=with_ws)
        assert st == 0
        for r in range(R_):
            np.testing.assert_array_equal(got[r], R.topk_select(x[r].astype(np.float64), k))


def test_topk_long_rows_tie_group_at_threshold(cuda):
    """Long rows on the streaming path whose k-th value is shared by eight keys: the selection takes
    one, three, four or all eight of them, always the lowest indices of the group (the tie rule):
    the threshold either splits the group by index or takes it whole.  Bit-exact."""
    S = lib()
    g = synth.rng_for(78)
    R_, n, k = 4, 131072, 40000
    x = g.random((R_, n)).astype(np.float32)
    for r, takes in enumerate((1, 8, 4, 3)):
        v = np.sort(x[r])[::-1][k - takes]
        below = np.flatnonzero(x[r] < v)
        x[r, g.choice(below, size=7, replace=False)] = v       # eight keys now hold v
    got, _, st = _topk_gpu(S, x, k)
    assert st == 0
    for r in range(R_):
        np.testing.assert_array_equal(got[r], R.topk_select(x[r].astype(np.float64), k))


def test_topk_long_rows_crowded_threshold_sub_bin(cuda):
    """Long rows on the streaming path whose threshold sub-bin holds between 1024 and 8192
    candidates, so the resolve step takes its 64-bit digit search (and marks the selected ones
    there): 3000 keys sharing the k-th value (rows 0-1, the group split at different offsets), or
    3000 distinct values 1e-7 apart (about 1.7 float32 ulps at 0.6), a span of 3e-4 against a
    sub-bin width near 1e-3, around the k-th value (rows 2-3).  The window (about 3.3 % of 262144 keys) plus the group stays inside the candidate
    list (16384).  Bit-exact against the oracle."""
    S = lib()
    g = synth.rng_for(80)
    R_, n, k = 4, 262144, 100000
    x = g.random((R_, n)).astype(np.float32)
    for r in range(R_):
        order = np.argsort(-x[r].astype(np.float64), kind="stable")
        v = x[r, order[k - 1]]
        lo = max(0, k - 1 - (500 if r % 2 == 0 else 2500))
        grp = order[lo:lo + 3000]                        # 3000 keys ranked around the k-th
        if r < 2:
            x[r, grp] = v                                 # one tie group holding the threshold
        else:
            x[r, grp] = (v.astype(np.float64) + (np.arange(3000) - 1500) * 1e-7).astype(np.float32)
    got, _, st = _topk_gpu(S, x, k)
    assert st == 0
    for r in range(R_):
        np.testing.assert_array_equal(got[r], R.topk_select(x[r].astype(np.float64), k))


def test_topk_long_rows_special_values_and_strides(cuda):
    """Long rows (n = 100003: a ragged last chunk) with special values, bit-exact against the
    oracle for k from 1 to n - 7:
    - row 0: 50 keys each of +inf and -inf (tie groups at the very top and bottom);
    - row 1: half the keys zeros of either sign (-0.0 equals +0.0; a tie group of 50 K keys);
    - row 2: denormals only;
    - row 3: lognormal.
    The row stride 100008 keeps the streaming path; the stride 100005 (not a multiple of 4) takes
    the cluster kernel; the results agree."""
    S = lib()
    g = synth.rng_for(79)
    R_, n = 4, 100003
    x = g.standard_normal((R_, n)).astype(np.float32)
    x[0, g.choice(n, 50, replace=False)] = np.inf
    x[0, g.choice(n, 50, replace=False)] = -np.inf
    z = g.choice(n, n // 2, replace=False)
    x[1, z] = np.where(g.random(z.size) < 0.5, -0.0, 0.0).astype(np.float32)
    x[2] = (g.standard_normal(n) * 1e-39).astype(np.float32)
    x[3] = g.lognormal(0.0, 2.0, n).astype(np.float32)
    want = {k: [R.topk_select(x[r].astype(np.float64), k) for r in range(R_)] for k in (1, 3000, n // 2, n - 7)}
    for ld in (100008, 100005):
        buf = np.zeros((R_, ld), np.float32)
        buf[:, :n] = x
        sc = to_dev(buf)
        for k, rows in want.items():
            out = torch.full((R_, k), -1, dtype=torch.int32, device="cuda")
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            nb = S.topk_workspace_size(R_, n, k)
            ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
            S.topk_select(sc, R_, n, ld, k, out, k, ws=ws, ws_bytes=nb, dev_status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            got = out.cpu().numpy()
            for r in range(R_):
                np.testing.assert_array_equal(got[r], rows[r], err_msg=f"ld {ld} k {k} row {r}")


# ------------------------------------------------------------------------------------------------
# K5 gather
# ------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("row_bytes,align16", [(4, True), (12, False), (1536, True), (1540, False), (8192, True)])
def test_gather_rows_and_compose(cuda, row_bytes, align16):
    S = lib()
    g = synth.rng_for(row_bytes)
    Rr, n, k = 5, 300, 123
    words = row_bytes // 4
    src = g.integers(-2**31, 2**31 - 1, (Rr, n, words), dtype=np.int64).astype(np.int32)
    idx = np.stack([np.sort(g.choice(n, k, replace=False)) for _ in range(Rr)]).astype(np.int32)
    comp_in = g.integers(0, 10**6, (Rr, n)).astype(np.int32)
    s = to_dev(src, torch.int32)
    d = torch.zeros((Rr, k, words), dtype=torch.int32, device="cuda")
    co = torch.zeros((Rr, k), dtype=torch.int32, device="cuda")
    S.gather_kept(s, n * row_bytes, row_bytes, n, row_bytes, Rr, to_dev(idx, torch.int32), k, k, d, k * row_bytes,
                  row_bytes, compose_in=to_dev(comp_in, torch.int32), ld_compose=n, compose_out=co)
    torch.cuda.synchronize()
    want = np.stack([src[r][idx[r]] for r in range(Rr)])
    np.testing.assert_array_equal(d.cpu().numpy(), want)
    np.testing.assert_array_equal(co.cpu().numpy(), np.stack([comp_in[r][idx[r]] for r in range(Rr)]))


def test_gather_checked_index_reports(cuda):
    S = lib()
    src = to_dev(np.arange(40, dtype=np.int32).reshape(1, 10, 4), torch.int32)
    idx = to_dev(np.array([[1, 3, 12]], np.int32), torch.int32)
    d = torch.zeros((1, 3, 4), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.gather_kept(src, 160, 16, 10, 16, 1, idx, 3, 3, d, 48, 16, check_index=1, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == S.E_INDEX
    np.testing.assert_array_equal(d.cpu().numpy()[0, :2], np.arange(40).reshape(10, 4)[[1, 3]])
