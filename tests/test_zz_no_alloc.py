"""The attention entry point for callers that cannot allocate (library-owned scratch).

Some callers of this library cannot allocate device memory -- a plugin whose host application
owns every allocation, a real-time loop that must stay out of the CUDA allocator -- so they use
spatten_attention_layer_noalloc, which keeps its scratch in a fixed device array inside the
library.  This test calls it through the C ABI:

* first on a different, larger problem (another seed, shape and threshold, with many refetched
  rows), which leaves that problem's partial sums in the shared array;
* then twice on the target problem.  Both calls must give results bit-identical to the workspace
  entry point spatten_attention_layer on the same inputs (the kernels and the reduction order are
  the same, so nothing may differ): a partial sum that a call read without writing it first would
  still hold the other problem's value and show up here.  The target is also checked once against
  the oracle with the tolerances of the other attention tests.

It also checks that a problem too large for the fixed array is refused before anything runs.  It
lives in its own file, collected last, and needs no state from other tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from gpu_helpers import BF, lib, to_dev, ws
from test_gpu_attention import check, make_layer, oracle_layer

pytestmark = pytest.mark.gpu


class Problem:
    """One attention layer over device-quantized K/V with every output buffer, set up through the
    C ABI (spatten_quantize_kv), as a caller without an allocator would be handed it."""

    def __init__(self, S, B, H, n, d, theta, seed, boost, keep):
        self.B, self.H, self.n, self.d, self.theta = B, H, n, d, theta
        self.raw, self.gain = make_layer(B, H, n, d, seed=seed, boost=boost)
        self.heads = np.array([keep] * B, np.int32)
        HD = H * d
        x = to_dev(self.raw, BF)
        self.x = x
        self.head_dev = to_dev(self.heads, torch.int32)
        a = S.attn_args()
        a.B, a.H, a.n_q, a.n_kv, a.d_h, a.H_kept = B, H, n, n, d, len(keep)
        a.head_idx, a.head_idx_ld = self.head_dev.data_ptr(), len(keep)
        a.q, a.q_dtype, a.q_ld_tok = x.data_ptr(), S.BF16, 3 * HD
        a.quantized, a.kv_cap = 1, n
        self.planes = {}
        for t, name in ((0, "k"), (1, "v")):
            msb = torch.empty((B, H, n, d), dtype=torch.int8, device="cuda")
            lsb = torch.empty((B, H, n, d // 2), dtype=torch.uint8, device="cuda")
            sc = torch.empty(B * H, device="cuda")
            S.quantize_kv(x.data_ptr() + (t + 1) * HD * 2, B, H, n, d, 3 * HD, msb, lsb, n, 0, scale_out=sc,
                          row_gain=to_dev(self.gain) if t == 0 else None, ld_gain=n, dtype=S.BF16)
            self.planes[name] = (msb, lsb, sc)
            setattr(a, f"{name}_msb", msb.data_ptr())
            setattr(a, f"{name}_lsb", lsb.data_ptr())
            setattr(a, f"{name}_scale", sc.data_ptr())
        self.o = torch.empty((B, n, HD), dtype=BF, device="cuda")
        self.tok = torch.empty((B, n), device="cuda")
        self.head = torch.empty((B, H), device="cuda")
        self.flags = torch.empty((B, H, n), dtype=torch.uint8, device="cuda")
        self.count = torch.empty(1, dtype=torch.int32, device="cuda")
        a.o, a.o_ld_tok, a.zero_pruned_heads = self.o.data_ptr(), HD, 1
        a.tok_imp, a.tok_imp_ld, a.head_imp = self.tok.data_ptr(), n, self.head.data_ptr()
        a.refetch_flags, a.refetch_count = self.flags.data_ptr(), self.count.data_ptr()
        a.refetch_threshold = theta
        self.a = a

    def clear(self):
        """Outputs start from values no call writes (importance is accumulated with +=)."""
        self.o.fill_(3.0)
        self.tok.zero_()
        self.head.zero_()
        self.flags.fill_(7)
        self.count.zero_()

    def result(self):
        torch.cuda.synchronize()
        out = dict(o=self.o.float().cpu().numpy(), tok=self.tok.cpu().numpy(), head=self.head.cpu().numpy(),
                   flags=self.flags.cpu().numpy(), count=int(self.count.item()))
        mk, lk, sk = self.planes["k"]
        mv, lv, sv = self.planes["v"]
        out.update(msbk=mk.cpu().numpy(), lsbk=lk.cpu().numpy(), sk=sk.cpu().numpy().reshape(self.B, self.H),
                   msbv=mv.cpu().numpy(), lsbv=lv.cpu().numpy(), sv=sv.cpu().numpy().reshape(self.B, self.H))
        return out

    def run_workspace(self, S):
        self.clear()
        w = ws(S.attention_workspace_size(self.a))
        S.attention_layer(self.a, w, w.numel())
        return self.result()

    def run_noalloc(self, S):
        self.clear()
        status = S.lib.spatten_attention_layer_noalloc(C.byref(self.a), torch.cuda.current_stream().cuda_stream)
        assert status == S.OK, S.lib.spatten_status_string(status)
        return self.result()


def assert_identical(got, ref, what):
    for key in ("o", "tok", "head", "flags", "count"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=f"{what}: {key}")


def test_noalloc_bit_identical_to_workspace_entry_after_another_problem(cuda):
    S = lib()
    other = Problem(S, B=4, H=8, n=450, d=64, theta=0.4, seed=7, boost=20, keep=[0, 2, 3, 5, 6, 7])
    target = Problem(S, B=3, H=6, n=300, d=64, theta=0.1, seed=2024, boost=15, keep=[0, 2, 3, 5])
    for p in (other, target):
        assert 0 < S.attention_workspace_size(p.a) <= S.NOALLOC_SCRATCH_BYTES
    ref_other = other.run_workspace(S)
    ref = target.run_workspace(S)
    assert ref_other["count"] > 0 and ref["count"] > 0          # both problems refetch rows
    # the other problem fills the shared scratch first
    assert_identical(other.run_noalloc(S), ref_other, "other problem")
    for call in range(2):
        got = target.run_noalloc(S)
        assert_identical(got, ref, f"target, call {call}")
    # and the target against the oracle (the same criteria as the other attention tests)
    o_ref = oracle_layer(target.raw, target.gain, target.B, target.H, target.n, target.d, target.theta,
                         target.heads, BF, got)
    check(got, o_ref, target.heads, target.H, target.d, 2e-2, 1e-2, "bf16")


def test_noalloc_refuses_problems_beyond_its_scratch(cuda):
    S = lib()
    p = Problem(S, B=3, H=6, n=300, d=64, theta=0.1, seed=2024, boost=15, keep=[0, 2, 3, 5])
    a = p.a
    a.B = 64                      # scratch need grows with B; no kernel runs on refusal
    a.n_q = a.n_kv = a.kv_cap = a.tok_imp_ld = 4096
    assert S.attention_workspace_size(a) > S.NOALLOC_SCRATCH_BYTES
    status = S.lib.spatten_attention_layer_noalloc(C.byref(a), torch.cuda.current_stream().cuda_stream)
    assert status == S.E_WORKSPACE
