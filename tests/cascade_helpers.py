"""Run spatten_cascade_forward from a synthetic workload and bring every result to the host."""
import ctypes as C

import numpy as np
import torch

from gpu_helpers import BF, to_dev, ws


def upload_prefill(S, w, d, trace=True):
    dt = BF if w.dtype == "bf16" else torch.float32
    B, T, D, H, L = w.B, w.T, w.D, w.H, w.L
    HD = H * w.d_h
    X = to_dev(d["X"], dt)
    Wt = [(to_dev(d["w_qkv"][l], dt), to_dev(d["w_o"][l], dt)) for l in range(L)]
    gain = to_dev(d["key_gain"].astype(np.float32)) if d["key_gain"] is not None else None
    bufs = dict(X=X, W=Wt, gain=gain,
                x_out=torch.zeros((B, w.token_keep[-1], D), dtype=dt, device="cuda"),
                kept_tok=torch.full((L, B, T), -1, dtype=torch.int32, device="cuda"),
                kept_head=torch.full((L, B, H), -1, dtype=torch.int32, device="cuda"),
                tok_imp=torch.zeros((B, T), dtype=torch.float32, device="cuda"),
                head_imp=torch.zeros((B, H), dtype=torch.float32, device="cuda"),
                refetch=torch.zeros(L, dtype=torch.int32, device="cuda"),
                status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    if trace:
        bufs.update(tx=torch.zeros((L, B, T, D), dtype=dt, device="cuda"),
                    tqkv=torch.zeros((L, B, T, 3 * HD), dtype=dt, device="cuda"),
                    to=torch.zeros((L, B, T, HD), dtype=dt, device="cuda"),
                    ttok=torch.zeros((L, B, T), dtype=torch.float32, device="cuda"),
                    thead=torch.zeros((L, B, H), dtype=torch.float32, device="cuda"),
                    tflags=torch.zeros((L, B, H, T), dtype=torch.uint8, device="cuda"))
    cfg = S.make_cfg(S.PREFILL, B, T, D, H, w.d_h, L, S.BF16 if dt == BF else S.F32, w.token_keep, w.head_keep,
                     w.quant, w.theta)
    io = S.cascade_io()
    p = S.ptr
    io.x, io.key_gain, io.x_out = p(X), p(gain), p(bufs["x_out"])
    io.kept_tok, io.kept_head = p(bufs["kept_tok"]), p(bufs["kept_head"])
    io.tok_imp, io.head_imp, io.refetch_count = p(bufs["tok_imp"]), p(bufs["head_imp"]), p(bufs["refetch"])
    io.dev_status = p(bufs["status"])
    if trace:
        io.trace_x, io.trace_qkv, io.trace_o = p(bufs["tx"]), p(bufs["tqkv"]), p(bufs["to"])
        io.trace_tok_imp, io.trace_head_imp, io.trace_flags = p(bufs["ttok"]), p(bufs["thead"]), p(bufs["tflags"])
    wsb = ws(S.cascade_workspace_size(cfg))
    bufs.update(cfg=cfg, io=io, ws=wsb)
    return bufs


def run_prefill(S, bufs):
    S.cascade_forward(bufs["cfg"], bufs["W"], bufs["io"], bufs["ws"], bufs["ws"].numel())
    torch.cuda.synchronize()


def host(bufs):
    out = {}
    for k, v in bufs.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.float().cpu().numpy() if v.dtype in (BF, torch.float32) else v.cpu().numpy()
    return out
