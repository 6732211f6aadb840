"""Device state of a generation (decode) run: per-layer quantized K/V caches, the persistent token
importance, the weights, and one ``spatten_cascade_forward`` call per generated token.

Argument marshalling only -- the prompt caches are quantized by ``spatten_quantize_kv`` and every
step runs in the library's kernels.
"""
import ctypes as C

import numpy as np
import torch

from . import spatten as S
from .synth import DecodeWorkload, linear_decode_keep

_TORCH = {S.F32: torch.float32, S.BF16: torch.bfloat16}


class DecodeState:
    """Caches for ``cap`` rows per (sequence, head) and ``layers`` layers.

    ``prompt_k[l]`` / ``prompt_v[l]``: host float32 [B, H, T0, d_h] prompt keys and values, one
    amax scale per (sequence, head, tensor) computed on the device.  ``w_qkv[l]`` [D, 3*H*d_h] and
    ``w_o[l]`` [H*d_h, D] host arrays, cast to ``dtype`` on upload.
    """

    def __init__(self, w: DecodeWorkload, w_qkv, w_o, prompt_k, prompt_v, dtype=S.BF16, trace=False):
        self.w = w
        self.L = len(w_qkv)
        self.dtype = dtype
        tdt = _TORCH[dtype]
        B, H, dh, T0, cap = w.B, w.H, w.d_h, w.T0, w.cap
        HD = H * dh
        dev = "cuda"
        self.W = [(torch.from_numpy(np.ascontiguousarray(a)).to(tdt).to(dev),
                   torch.from_numpy(np.ascontiguousarray(b)).to(tdt).to(dev)) for a, b in zip(w_qkv, w_o)]
        self.caches = []
        for l in range(self.L):
            c = dict(k_msb=torch.zeros((B, H, cap, dh), dtype=torch.int8, device=dev),
                     k_lsb=torch.zeros((B, H, cap, dh // 2), dtype=torch.uint8, device=dev),
                     v_msb=torch.zeros((B, H, cap, dh), dtype=torch.int8, device=dev),
                     v_lsb=torch.zeros((B, H, cap, dh // 2), dtype=torch.uint8, device=dev),
                     k_scale=torch.zeros(B * H, dtype=torch.float32, device=dev),
                     v_scale=torch.zeros(B * H, dtype=torch.float32, device=dev))
            for key, src in (("k", prompt_k[l]), ("v", prompt_v[l])):
                # token-major [B, T0, H*d_h] rows, the layout the projections produce
                x = torch.from_numpy(np.ascontiguousarray(
                    np.asarray(src, np.float32).transpose(0, 2, 1, 3).reshape(B, T0, HD))).to(dev)
                S.quantize_kv(x, B, H, T0, dh, HD, c[key + "_msb"], c[key + "_lsb"], cap, 0,
                              scale_out=c[key + "_scale"], dtype=S.F32)
            self.caches.append(c)
        self.cache_arr = (S.decode_cache * self.L)(*[
            S.decode_cache(S.ptr(c["k_msb"]), S.ptr(c["k_lsb"]), S.ptr(c["k_scale"]),
                           S.ptr(c["v_msb"]), S.ptr(c["v_lsb"]), S.ptr(c["v_scale"])) for c in self.caches])
        self.n_old = T0
        self.x = torch.zeros((B, w.D), dtype=tdt, device=dev)
        self.x_out = torch.zeros((B, w.D), dtype=tdt, device=dev)
        self.kept_tok = torch.full((self.L, B, cap), -1, dtype=torch.int32, device=dev)
        self.tok_imp = torch.zeros((B, cap), dtype=torch.float32, device=dev)
        self.head_imp = torch.zeros((B, H), dtype=torch.float32, device=dev)
        self.refetch = torch.zeros(self.L, dtype=torch.int32, device=dev)
        self.sat = torch.zeros(1, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.trace = None
        if trace:
            self.trace = dict(x=torch.zeros((self.L, B, w.D), dtype=tdt, device=dev),
                              qkv=torch.zeros((self.L, B, 3 * HD), dtype=tdt, device=dev),
                              o=torch.zeros((self.L, B, HD), dtype=tdt, device=dev),
                              tok_imp=torch.zeros((self.L, B, cap), dtype=torch.float32, device=dev),
                              flags=torch.zeros((self.L, B, H), dtype=torch.uint8, device=dev))
        cfg = self.cfg_for(cap)
        self.ws = torch.empty(max(S.cascade_workspace_size(cfg), 256), dtype=torch.uint8, device=dev)

    def keep(self, n: int) -> list[int]:
        return linear_decode_keep(n, self.L)

    def cfg_for(self, n: int):
        w = self.w
        return S.make_cfg(S.DECODE_STEP, w.B, n, w.D, w.H, w.d_h, self.L, self.dtype, self.keep(n), None,
                          True, w.theta)

    def io(self, x=None, x_out=None, refetch=None, events=None):
        """The cascade_io of the next step; the optional device tensors replace this state's input
        row buffer, output row buffer and refetch counters, and `events` (a ctypes array of 2*L
        cudaEvent_t) times the attention launches."""
        io = S.cascade_io()
        p = S.ptr
        io.x = p(self.x if x is None else x)
        io.x_out = p(self.x_out if x_out is None else x_out)
        io.kept_tok = p(self.kept_tok)
        io.head_imp, io.sat_count = p(self.head_imp), p(self.sat)
        io.refetch_count = p(self.refetch if refetch is None else refetch)
        io.dev_status = p(self.status)
        io.caches = C.cast(self.cache_arr, C.POINTER(S.decode_cache))
        io.cap, io.n_old, io.dec_tok_imp = self.w.cap, self.n_old, p(self.tok_imp)
        if self.trace is not None:
            t = self.trace
            io.trace_x, io.trace_qkv, io.trace_o = p(t["x"]), p(t["qkv"]), p(t["o"])
            io.trace_tok_imp, io.trace_flags = p(t["tok_imp"]), p(t["flags"])
        if events is not None:
            io.attn_events = C.cast(events, C.POINTER(S.vp))
        return io

    def reset(self, n_old: int | None = None):
        """Rewind to `n_old` cache rows (default: the prompt) and clear the importance state; rows
        past n_old are overwritten by later steps.  Enqueued on the current stream."""
        self.n_old = self.w.T0 if n_old is None else n_old
        self.tok_imp.zero_()
        self.head_imp.zero_()
        self.sat.zero_()

    def step(self, x=None, x_out=None, refetch=None, events=None, stream=None):
        """Generate one token from the rows in ``x`` (default ``self.x``, which the caller fills):
        appends row n_old to every layer's cache, attends, and advances n_old."""
        if self.n_old >= self.w.cap:
            raise ValueError("decode cache is full")
        cfg = self.cfg_for(self.n_old + 1)
        S.cascade_forward(cfg, self.W, self.io(x, x_out, refetch, events), self.ws, self.ws.numel(), stream)
        self.n_old += 1
