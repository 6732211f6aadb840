"""Host-side checks of the C ABI (no GPU needed): the library loads and exports every function
include/spatten.h declares, the ctypes structs match the header's layout (checked by compiling a
C program against the header with gcc), and argument errors are reported before any launch."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spatten.h")


@pytest.fixture(scope="module")
def S():
    from cascade_token_head_b200 import build
    build.build()
    from cascade_token_head_b200 import spatten
    return spatten


def header_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(spatten_\w+)\s*\(", txt)))


def test_exports_every_declared_function(S):
    declared = header_functions()
    assert set(declared) == set(S.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", S.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (spatten_\w+)", out))
    assert set(declared) <= exported
    for name in declared:
        assert hasattr(S.lib, name)
    assert S.lib.spatten_abi_version() == 1


def test_selftest_exp2_poly_rejects_bad_arguments(S):
    L = S.lib
    assert L.spatten_selftest_exp2_poly(None, 16, 4, None) == S.E_ARG
    assert L.spatten_selftest_exp2_poly(16, None, 4, None) == S.E_ARG
    assert L.spatten_selftest_exp2_poly(16, 32, 0, None) == S.E_ARG


def test_struct_layout_matches_header(S, tmp_path):
    structs = {"spatten_attn_args": S.attn_args, "spatten_cascade_cfg": S.cascade_cfg,
               "spatten_layer_weights": S.layer_weights, "spatten_decode_cache": S.decode_cache,
               "spatten_cascade_io": S.cascade_io}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "spatten.h"', 'int main(void){']
    for cname, py in structs.items():
        lines.append(f'printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0;}")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for ln in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        s, f, v = ln.split()
        got[(s, f)] = int(v)
    for cname, py in structs.items():
        assert got[(cname, "sizeof")] == C.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)


def test_status_strings(S):
    for s in range(11):
        assert S.lib.spatten_status_string(s).decode().startswith("SPATTEN_")
    assert b"UNKNOWN" in S.lib.spatten_status_string(99)


def test_topk_argument_errors(S):
    L = S.lib
    assert L.spatten_topk_select(None, 1, 10, 10, 3, None, 0, 16, 3, None, None, 0, None, None) == S.E_ARG
    assert L.spatten_topk_select(16, 1, 10, 10, 11, None, 0, 16, 11, None, None, 0, None, None) == S.E_SHAPE
    assert L.spatten_topk_select(16, 1, 10, 5, 3, None, 0, 16, 3, None, None, 0, None, None) == S.E_SHAPE
    assert L.spatten_topk_select(16, 1, 10, 10, 3, None, 0, 16, 2, None, None, 0, None, None) == S.E_SHAPE
    assert L.spatten_topk_select(16, 0, 10, 10, 3, None, 0, 16, 3, None, None, 0, None, None) == S.E_ARG
    # composition needs a map
    assert L.spatten_topk_select(16, 1, 10, 10, 3, None, 0, 16, 3, 32, None, 0, None, None) == S.E_ARG


def test_topk_workspace_size_rules(S):
    """The optional top-k workspace: none below 64 K keys per row; from there, at least the
    candidate lists (8 bytes per candidate, max(4096, n/16) candidates per row) plus the per-chunk
    counters (8 K-key chunks) and the selection bit mask (one bit per key);
    linear in the row count; k does not matter; rows longer than 8192 chunks (64 M keys) take the
    cluster kernel and need none."""
    f = S.topk_workspace_size
    for n in (1, 1000, 65535):
        assert f(64, n, max(1, n // 2)) == 0
    for n in (65536, 262144, 1048576, 1 << 22):
        nchunk = -(-n // 8192)
        need = 64 * (max(4096, n // 16) * 8 + nchunk * (4 + 4 + 64 * 4 + 8192 // 8))
        b = f(64, n, n // 2)
        assert b >= need
        assert b == f(64, n, 1) == f(64, n, n - 1)
        assert f(128, n, 7) - b >= need - 256 * 16   # per-row parts (each region rounded to 256 B)
    assert f(1, 8192 * 8192, 5) > 0
    assert f(1, 8192 * 8192 + 1, 5) == 0


def test_quantize_argument_errors(S):
    L = S.lib
    q = L.spatten_quantize_kv
    assert q(None, 1, 1, 1, 4, 64, 64, None, 0, None, 16, 16, 4, 0, 16, None, None) == S.E_ARG
    assert q(16, 1, 1, 1, 4, 60, 64, None, 0, None, 16, 16, 4, 0, 16, None, None) == S.E_ARG   # d_h % 8
    assert q(16, 1, 1, 1, 4, 64, 64, None, 0, None, 16, 16, 4, 1, 16, None, None) == S.E_SHAPE  # row0+n > cap
    assert q(17, 1, 1, 1, 4, 64, 64, None, 0, None, 16, 16, 4, 0, 16, None, None) == S.E_ALIGN
    assert q(16, 1, 1, 1, 4, 64, 68, None, 0, None, 16, 16, 4, 0, 16, None, None) == S.E_ALIGN  # ld*2 % 16
    assert q(16, 1, 1, 1, 4, 64, 64, None, 0, None, 16, 16, 4, 0, None, None, None) == S.E_ARG  # no scale out
    assert q(16, 7, 1, 1, 4, 64, 64, None, 0, None, 16, 16, 4, 0, 16, None, None) == S.E_ARG   # dtype


def test_gather_argument_errors(S):
    g = S.lib.spatten_gather_kept
    assert g(16, 0, 16, 4, 6, 1, 16, 4, 2, 32, 0, 16, None, 0, None, 0, None, None) == S.E_ARG   # row_bytes % 4
    assert g(16, 0, 16, 4, 16, 1, 16, 1, 2, 32, 0, 16, None, 0, None, 0, None, None) == S.E_SHAPE
    assert g(18, 0, 16, 4, 16, 1, 16, 4, 2, 32, 0, 16, None, 0, None, 0, None, None) == S.E_ALIGN
    assert g(16, 0, 16, 4, 16, 1, 16, 4, 2, 32, 0, 16, 64, 4, None, 0, None, None) == S.E_ARG   # half a compose pair
    assert g(16, 0, 16, 4, 16, 1, 16, 4, 0, 32, 0, 16, None, 0, None, 0, None, None) == S.OK    # k = 0: nothing


def _attn(S, **over):
    a = S.attn_args()
    a.B, a.H, a.n_q, a.n_kv, a.d_h, a.H_kept = 2, 4, 100, 100, 64, 4
    a.q, a.q_dtype, a.q_ld_tok = 1 << 20, S.BF16, 3 * 256
    a.quantized = 1
    a.k_msb = a.v_msb = a.k_lsb = a.v_lsb = 1 << 21
    a.k_scale = a.v_scale = 1 << 22
    a.kv_cap = 100
    a.o, a.o_ld_tok = 1 << 23, 256
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_attention_argument_errors_and_workspace(S):
    L = S.lib
    assert L.spatten_attention_workspace_size(C.byref(_attn(S))) > 0
    for over, want in [(dict(d_h=96), S.E_UNSUPPORTED), (dict(H_kept=5), S.E_ARG), (dict(H_kept=3), S.E_ARG),
                       (dict(q=0), S.E_ARG), (dict(q_ld_tok=100), S.E_SHAPE), (dict(kv_cap=50), S.E_SHAPE),
                       (dict(q=(1 << 20) + 8), S.E_ALIGN), (dict(kernel=9), S.E_ARG), (dict(kernel=5), S.E_ARG), (dict(v_keep=-1), S.E_ARG)]:
        assert L.spatten_attention_layer(C.byref(_attn(S, **over)), 1 << 24, 1 << 30, None) == want, over
    # workspace too small
    assert L.spatten_attention_layer(C.byref(_attn(S)), 1 << 24, 16, None) == S.E_WORKSPACE
    # local value pruning needs room for the per-head column sums, kept lists and V mask; keeping
    # every key (v_keep >= n_kv) is no pruning and needs nothing more
    base = L.spatten_attention_workspace_size(C.byref(_attn(S)))
    assert L.spatten_attention_workspace_size(C.byref(_attn(S, v_keep=50))) >= base + 2 * 4 * 100 * (4 + 1) + 2 * 4 * 50 * 4
    assert L.spatten_attention_workspace_size(C.byref(_attn(S, v_keep=100))) == base
    # a forced kernel that cannot run the problem
    assert L.spatten_attention_layer(C.byref(_attn(S, kernel=S.ATTN_DECODE)), 1 << 24, 1 << 30, None) == S.E_UNSUPPORTED
    assert (L.spatten_attention_layer(C.byref(_attn(S, kernel=S.ATTN_DECODE_PREDICATED)), 1 << 24, 1 << 30, None)
            == S.E_UNSUPPORTED)
    # the predicated decode form keeps one refetch flag per (sequence, kept head) when theta > 0
    size = lambda **o: L.spatten_attention_workspace_size(C.byref(_attn(S, n_q=1, **o)))
    single = size(kernel=S.ATTN_DECODE, refetch_threshold=0.1)
    assert size(kernel=S.ATTN_DECODE_PREDICATED, refetch_threshold=0.1) >= single + 2 * 4 * 4
    assert size(kernel=S.ATTN_DECODE_PREDICATED, refetch_threshold=0.0) == size(kernel=S.ATTN_DECODE, refetch_threshold=0.0)


def test_cascade_cfg_checks_and_workspace(S):
    from cascade_token_head_b200 import synth
    w = synth.bert_base_prefill()
    cfg = S.make_cfg(S.PREFILL, w.B, w.T, w.D, w.H, w.d_h, w.L, S.BF16, w.token_keep, w.head_keep, True, w.theta)
    n = S.cascade_workspace_size(cfg)
    assert n > 32 << 20
    bad = S.make_cfg(S.PREFILL, w.B, w.T, w.D, w.H, w.d_h, w.L, S.BF16, [w.T + 1] + w.token_keep[1:], w.head_keep,
                     True, w.theta)
    assert S.cascade_workspace_size(bad) == 0
    bad = S.make_cfg(S.PREFILL, w.B, w.T, w.D, w.H, w.d_h, w.L, S.BF16, w.token_keep, [12, 13] + w.head_keep[2:],
                     True, w.theta)
    assert S.cascade_workspace_size(bad) == 0
    dec = S.make_cfg(S.DECODE_STEP, 16, 1025, 1024, 16, 64, 24, S.BF16, synth.linear_decode_keep(1025, 24), None,
                     False, 0.2)
    assert S.cascade_workspace_size(dec) == 0       # decode needs the quantized cache
