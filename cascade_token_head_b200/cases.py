"""Run one library kernel on a seeded synthetic case (for profiling and per-kernel timing).

    python -m cascade_token_head_b200.cases attention --B 32 --H 12 --n 512 --d 64 --theta 0.1 --reps 3
    python -m cascade_token_head_b200.cases topk --R 64 --n 1048576 --k 524288 --reps 3
    python -m cascade_token_head_b200.cases decode --B 16 --H 16 --n 1152 --keep 576 --reps 3
    python -m cascade_token_head_b200.cases decode_step --reps 4
    python -m cascade_token_head_b200.cases quantize --B 32 --H 12 --n 512 --d 64 --reps 3
    python -m cascade_token_head_b200.cases gather --B 32 --n 512 --k 461 --row-bytes 1536 --reps 3

Each prints one JSON line with the mean CUDA-event time per call and the algorithmic bytes or
flops of one call.  Inputs are drawn on the host from a seeded generator and copied once.
"""
from __future__ import annotations

import argparse
import json
import math

import numpy as np
import torch

from . import spatten as S
from . import synth


def _time(fn, reps: int) -> float:
    """Mean device time of one call: `reps` calls captured in a CUDA graph and replayed (host launch
    overhead excluded; for small kernels it would otherwise be what is timed)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def attention_case(B, H, n, d, theta, boost, kernel, reps, n_kv=None):
    g = synth.rng_for(7)
    HD = H * d
    x = torch.from_numpy(g.standard_normal((B, n, 3 * HD))).to(torch.bfloat16).cuda()
    gain = np.ones((B, n), np.float32)
    for b in range(B):
        gain[b, g.choice(n, max(1, int(boost * n)), replace=False)] = 4.0
    gain = torch.from_numpy(gain).cuda()
    planes = []
    for t in range(2):
        msb = torch.empty((B, H, n, d), dtype=torch.int8, device="cuda")
        lsb = torch.empty((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
        sc = torch.empty(B * H, device="cuda")
        S.quantize_kv(x.data_ptr() + (t + 1) * HD * 2, B, H, n, d, 3 * HD, msb, lsb, n, 0, scale_out=sc,
                      row_gain=gain if t == 0 else None, ld_gain=n, dtype=S.BF16)
        planes.append((msb, lsb, sc))
    a = S.attn_args()
    a.B, a.H, a.n_q, a.n_kv, a.d_h, a.H_kept = B, H, n, n, d, H
    a.q, a.q_dtype, a.q_ld_tok = x.data_ptr(), S.BF16, 3 * HD
    a.quantized, a.kv_cap = 1, n
    (km, kl, ks), (vm, vl, vsc) = planes
    a.k_msb, a.k_lsb, a.k_scale = km.data_ptr(), kl.data_ptr(), ks.data_ptr()
    a.v_msb, a.v_lsb, a.v_scale = vm.data_ptr(), vl.data_ptr(), vsc.data_ptr()
    o = torch.empty((B, n, HD), dtype=torch.bfloat16, device="cuda")
    tok = torch.zeros((B, n), device="cuda")
    head = torch.zeros((B, H), device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    a.o, a.o_ld_tok = o.data_ptr(), HD
    a.tok_imp, a.tok_imp_ld, a.head_imp, a.refetch_count = tok.data_ptr(), n, head.data_ptr(), cnt.data_ptr()
    a.refetch_threshold, a.kernel = theta, kernel
    ws = torch.empty(S.attention_workspace_size(a), dtype=torch.uint8, device="cuda")
    ms = _time(lambda: S.attention_layer(a, ws, ws.numel()), reps)
    flops = 4.0 * B * H * n * n * d
    return dict(case="attention", B=B, H=H, n=n, d=d, theta=theta, ms=ms, flops=flops,
                tflops=flops / ms / 1e9, refetch_rows=int(cnt.item()) // (2 * reps + 1))


def topk_case(R, n, k, dist, reps):
    x = torch.from_numpy(synth.draw_topk_row_block(R, n, dist, 0.01, seed=3)).cuda()
    out = torch.empty((R, max(k, 1)), dtype=torch.int32, device="cuda")
    nb = S.topk_workspace_size(R, n, k)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    ms = _time(lambda: S.topk_select(x, R, n, n, k, out, max(k, 1), ws=ws, ws_bytes=nb), reps)
    byts = R * (4.0 * n + 4.0 * k)
    return dict(case="topk", R=R, n=n, k=k, dist=dist, ms=ms, bytes=byts, gbs=byts / ms / 1e6)


def gather_case(B, n, k, row_bytes, reps):
    g = synth.rng_for(5)
    src = torch.empty((B, n, row_bytes), dtype=torch.uint8, device="cuda").random_(0, 255)
    idx = torch.from_numpy(np.stack([np.sort(g.choice(n, k, replace=False)) for _ in range(B)]).astype(np.int32)).cuda()
    dst = torch.empty((B, k, row_bytes), dtype=torch.uint8, device="cuda")
    ms = _time(lambda: S.gather_kept(src, n * row_bytes, row_bytes, n, row_bytes, B, idx, k, k, dst, k * row_bytes,
                                     row_bytes), reps)
    byts = B * (2.0 * k * row_bytes + 4.0 * k)
    return dict(case="gather", B=B, n=n, k=k, row_bytes=row_bytes, ms=ms, bytes=byts, gbs=byts / ms / 1e6)


def quantize_case(B, H, n, d, reps):
    g = synth.rng_for(9)
    HD = H * d
    x = torch.from_numpy(g.standard_normal((B, n, 3 * HD))).to(torch.bfloat16).cuda()
    msb = torch.empty((B, H, n, d), dtype=torch.int8, device="cuda")
    lsb = torch.empty((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
    sc = torch.empty(B * H, device="cuda")
    ms = _time(lambda: S.quantize_kv(x.data_ptr() + HD * 2, B, H, n, d, 3 * HD, msb, lsb, n, 0, scale_out=sc,
                                     dtype=S.BF16), reps)
    byts = B * H * n * d * (2.0 + 1.0 + 0.5)
    return dict(case="quantize", B=B, H=H, n=n, d=d, ms=ms, bytes=byts, gbs=byts / ms / 1e6)


def decode_case(B, H, n, d, keep, theta, reps, kernel=0):
    g = synth.rng_for(11)
    HD = H * d
    kv = torch.from_numpy(g.standard_normal((B, n, 3 * HD))).to(torch.bfloat16).cuda()
    q = kv[:, :1, :].contiguous()
    planes = []
    for t in range(2):
        msb = torch.empty((B, H, n, d), dtype=torch.int8, device="cuda")
        lsb = torch.empty((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
        sc = torch.empty(B * H, device="cuda")
        S.quantize_kv(kv.data_ptr() + (t + 1) * HD * 2, B, H, n, d, 3 * HD, msb, lsb, n, 0, scale_out=sc, dtype=S.BF16)
        planes.append((msb, lsb, sc))
    idx = torch.from_numpy(np.stack([np.sort(g.choice(n, keep, replace=False)) for _ in range(B)]).astype(np.int32)).cuda()
    a = S.attn_args()
    a.B, a.H, a.n_q, a.n_kv, a.d_h, a.H_kept = B, H, 1, keep, d, H
    a.q, a.q_dtype, a.q_ld_tok = q.data_ptr(), S.BF16, 3 * HD
    a.quantized, a.kv_cap = 1, n
    (km, kl, ks), (vm, vl, vsc) = planes
    a.k_msb, a.k_lsb, a.k_scale = km.data_ptr(), kl.data_ptr(), ks.data_ptr()
    a.v_msb, a.v_lsb, a.v_scale = vm.data_ptr(), vl.data_ptr(), vsc.data_ptr()
    a.kv_idx, a.kv_idx_ld = idx.data_ptr(), keep
    o = torch.empty((B, 1, HD), dtype=torch.bfloat16, device="cuda")
    tok = torch.zeros((B, n), device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    a.o, a.o_ld_tok, a.tok_imp, a.tok_imp_ld = o.data_ptr(), HD, tok.data_ptr(), n
    a.tok_imp_map, a.tok_imp_map_ld, a.refetch_count = idx.data_ptr(), keep, cnt.data_ptr()
    a.refetch_threshold, a.kernel = theta, kernel
    ws = torch.empty(S.attention_workspace_size(a), dtype=torch.uint8, device="cuda")
    ms = _time(lambda: S.attention_layer(a, ws, ws.numel()), reps)
    refetched = int(cnt.item()) / (2 * reps + 1)
    byts = B * H * keep * d * 2.0 + refetched * keep * d + B * keep * 4.0
    return dict(case="decode", B=B, H=H, n=n, keep=keep, d=d, kernel=kernel, theta=theta, ms=ms, bytes=byts, gbs=byts / ms / 1e6,
                refetch_frac=refetched / (B * H))


def decode_step_case(reps, steps_done=0):
    """Generated tokens of the GPT-2-medium decode workload (B=16 after a 1024-token prompt, 24
    layers): one spatten_cascade_forward per token, after `steps_done` earlier tokens."""
    from .decode import DecodeState
    w = synth.gpt2m_decode()
    d = synth.draw_decode(w, steps=steps_done + 2 * reps + 2)
    st = DecodeState(w, d["w_qkv"], d["w_o"], d["k_prompt"], d["v_prompt"])
    xs = torch.from_numpy(d["x_steps"]).to(torch.bfloat16).cuda()
    for s in range(steps_done):
        st.step(x=xs[s])
    torch.cuda.synchronize()
    n0 = st.n_old
    # the same `reps` tokens, captured once and replayed: each replay rewinds to n0 first
    def tokens():
        st.reset(n0)
        for s in range(reps):
            st.step(x=xs[steps_done + s])
    ms = _time(tokens, 1) / reps
    assert int(st.status.item()) == 0
    return dict(case="decode_step", B=w.B, layers=w.L, cache_rows=n0 + 1, ms_per_token=ms,
                tokens_per_s=w.B / ms * 1e3)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["attention", "topk", "gather", "quantize", "decode", "decode_step"])
    ap.add_argument("--B", type=int, default=32)
    ap.add_argument("--H", type=int, default=12)
    ap.add_argument("--n", type=int, default=512)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--k", type=int, default=256)
    ap.add_argument("--R", type=int, default=64)
    ap.add_argument("--keep", type=int, default=576)
    ap.add_argument("--row-bytes", type=int, default=1536)
    ap.add_argument("--theta", type=float, default=0.1)
    ap.add_argument("--boost", type=float, default=0.05)
    ap.add_argument("--kernel", type=int, default=0)
    ap.add_argument("--dist", default="uniform")
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    if a.case == "attention":
        r = attention_case(a.B, a.H, a.n, a.d, a.theta, a.boost, a.kernel, a.reps)
    elif a.case == "topk":
        r = topk_case(a.R, a.n, a.k, a.dist, a.reps)
    elif a.case == "gather":
        r = gather_case(a.B, a.n, a.k, a.row_bytes, a.reps)
    elif a.case == "quantize":
        r = quantize_case(a.B, a.H, a.n, a.d, a.reps)
    elif a.case == "decode":
        r = decode_case(a.B, a.H, a.n, a.d, a.keep, a.theta, a.reps, a.kernel)
    else:
        r = decode_step_case(a.reps)
    print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
