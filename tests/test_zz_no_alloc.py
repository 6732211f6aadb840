"""The attention entry point for callers that cannot allocate (library-owned scratch).

Some callers of this library cannot allocate device memory -- a plugin whose host application
owns every allocation, a real-time loop that must stay out of the CUDA allocator -- so they use
spatten_attention_layer_noalloc, which keeps its scratch in a fixed device array inside the
library.  This test calls it through the C ABI twice in a row and checks each result against the
workspace entry point spatten_attention_layer on the same inputs, with the tolerances the other
attention tests use; it also checks that a problem too large for the fixed array is refused
before anything runs.  It lives in its own file, collected last, and needs no state from other
tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from cascade_token_head_b200 import synth

from gpu_helpers import BF, assert_close_bf16_out, lib, ws

pytestmark = pytest.mark.gpu


def _setup(S, B, H, n, d, theta):
    g = synth.rng_for(2024)
    HD = H * d
    x = torch.from_numpy(g.standard_normal((B, n, 3 * HD))).to(BF).cuda()
    gain = np.ones((B, n), np.float32)
    for b in range(B):
        gain[b, g.choice(n, max(1, n // 20), replace=False)] = 4.0
    gain = torch.from_numpy(gain).cuda()
    keep = np.array([[h for h in range(H) if h % 3 != 1] for _ in range(B)], np.int32)
    heads = torch.from_numpy(keep).cuda()
    bufs = dict(x=x, gain=gain, heads=heads)
    a = S.attn_args()
    a.B, a.H, a.n_q, a.n_kv, a.d_h, a.H_kept = B, H, n, n, d, keep.shape[1]
    a.head_idx, a.head_idx_ld = heads.data_ptr(), keep.shape[1]
    a.q, a.q_dtype, a.q_ld_tok = x.data_ptr(), S.BF16, 3 * HD
    a.quantized, a.kv_cap = 1, n
    for t, name in ((0, "k"), (1, "v")):
        msb = torch.empty((B, H, n, d), dtype=torch.int8, device="cuda")
        lsb = torch.empty((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
        sc = torch.empty(B * H, device="cuda")
        S.quantize_kv(x.data_ptr() + (t + 1) * HD * 2, B, H, n, d, 3 * HD, msb, lsb, n, 0, scale_out=sc,
                      row_gain=gain if t == 0 else None, ld_gain=n, dtype=S.BF16)
        bufs[name] = (msb, lsb, sc)
        setattr(a, f"{name}_msb", msb.data_ptr())
        setattr(a, f"{name}_lsb", lsb.data_ptr())
        setattr(a, f"{name}_scale", sc.data_ptr())
    bufs["o"] = torch.empty((B, n, HD), dtype=BF, device="cuda")
    bufs["tok"] = torch.empty((B, n), device="cuda")
    bufs["head"] = torch.empty((B, H), device="cuda")
    bufs["flags"] = torch.empty((B, H, n), dtype=torch.uint8, device="cuda")
    a.o, a.o_ld_tok, a.zero_pruned_heads = bufs["o"].data_ptr(), HD, 1
    a.tok_imp, a.tok_imp_ld, a.head_imp = bufs["tok"].data_ptr(), n, bufs["head"].data_ptr()
    a.refetch_flags = bufs["flags"].data_ptr()
    a.refetch_threshold = theta
    return a, bufs


def _clear(bufs):
    bufs["o"].fill_(3.0)
    bufs["tok"].zero_()
    bufs["head"].zero_()
    bufs["flags"].fill_(7)


def _result(bufs):
    torch.cuda.synchronize()
    return {k: bufs[k].float().cpu().numpy() for k in ("o", "tok", "head", "flags")}


def test_noalloc_matches_workspace_entry_on_two_calls(cuda):
    S = lib()
    a, bufs = _setup(S, B=3, H=6, n=300, d=64, theta=0.1)
    need = S.attention_workspace_size(a)
    assert 0 < need <= S.NOALLOC_SCRATCH_BYTES
    _clear(bufs)
    w = ws(need)
    S.attention_layer(a, w, w.numel())
    ref = _result(bufs)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        _clear(bufs)
        status = S.lib.spatten_attention_layer_noalloc(C.byref(a), stream)
        assert status == S.OK, S.lib.spatten_status_string(status)
        got = _result(bufs)
        assert_close_bf16_out(got["o"], ref["o"], 2e-2, "O (no-alloc vs workspace entry)")
        np.testing.assert_allclose(got["tok"], ref["tok"], rtol=0, atol=2e-5 * np.abs(ref["tok"]).max())
        np.testing.assert_allclose(got["head"], ref["head"], rtol=1e-2, atol=1e-6)
        np.testing.assert_array_equal(got["flags"], ref["flags"])
        kept = [h for h in range(6) if h % 3 != 1]
        assert ref["flags"][:, kept].max() <= 1 and ref["tok"].sum() > 0


def test_noalloc_refuses_problems_beyond_its_scratch(cuda):
    S = lib()
    a, bufs = _setup(S, B=3, H=6, n=300, d=64, theta=0.1)
    a.B = 64                      # scratch need grows with B; no kernel runs on refusal
    a.n_q = a.n_kv = a.kv_cap = a.tok_imp_ld = 4096
    assert S.attention_workspace_size(a) > S.NOALLOC_SCRATCH_BYTES
    status = S.lib.spatten_attention_layer_noalloc(C.byref(a), torch.cuda.current_stream().cuda_stream)
    assert status == S.E_WORKSPACE
