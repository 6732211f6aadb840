"""Thin ctypes binding of libspatten.so (include/spatten.h).  Argument marshalling only: every step
of the computation runs in the library's CUDA kernels (and cuBLASLt for the FC projections).

Importing this module loads the library and raises ImportError if it has not been built
(``python -m cascade_token_head_b200.build``); there is no fallback implementation.
Functions take torch tensors (device memory) or raw integer pointers, and run on torch's current
CUDA stream unless a stream is given.  Each returns None and raises SpattenError on a non-OK
status.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspatten.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m cascade_token_head_b200.build`")
lib = C.CDLL(LIB_PATH)

# ---- enums (spatten.h) --------------------------------------------------------------------------
OK, E_ARG, E_SHAPE, E_ALIGN, E_WORKSPACE, E_NONFINITE, E_CUDA, E_TIMEOUT, E_UNSUPPORTED, E_INDEX, E_RANGE = range(11)
F32, BF16 = 0, 1
PREFILL, DECODE_STEP = 0, 1
ATTN_AUTO, ATTN_CUDA_CORE, ATTN_TENSOR_CORE, ATTN_DECODE, ATTN_DECODE_PREDICATED = 0, 1, 2, 3, 4
MAX_LAYERS = 64

vp, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t


class attn_args(C.Structure):
    _fields_ = [("B", i32), ("H", i32), ("n_q", i32), ("n_kv", i32), ("d_h", i32), ("H_kept", i32),
                ("head_idx", vp), ("head_idx_ld", i64),
                ("q", vp), ("q_dtype", i32), ("q_ld_tok", i64),
                ("quantized", i32), ("k_msb", vp), ("k_lsb", vp), ("k_scale", vp),
                ("v_msb", vp), ("v_lsb", vp), ("v_scale", vp), ("kv_cap", i32),
                ("k", vp), ("v", vp), ("kv_dtype", i32), ("kv_ld_tok", i64),
                ("kv_idx", vp), ("kv_idx_ld", i64),
                ("sm_scale", f32), ("refetch_threshold", f32),
                ("o", vp), ("o_ld_tok", i64), ("zero_pruned_heads", i32),
                ("tok_imp", vp), ("tok_imp_ld", i64), ("tok_imp_map", vp), ("tok_imp_map_ld", i64),
                ("head_imp", vp), ("refetch_flags", vp), ("refetch_flags_ld", i64), ("refetch_count", vp),
                ("dev_status", vp),
                ("kernel", i32), ("v_keep", i32)]


class cascade_cfg(C.Structure):
    _fields_ = [("mode", i32), ("B", i32), ("T", i32), ("D", i32), ("H", i32), ("d_h", i32), ("L", i32),
                ("dtype", i32), ("token_keep", i32 * MAX_LAYERS), ("head_keep", i32 * MAX_LAYERS),
                ("quant", i32), ("refetch_threshold", f32), ("sm_scale", f32)]


class layer_weights(C.Structure):
    _fields_ = [("w_qkv", vp), ("w_o", vp)]


class decode_cache(C.Structure):
    _fields_ = [("k_msb", vp), ("k_lsb", vp), ("k_scale", vp), ("v_msb", vp), ("v_lsb", vp), ("v_scale", vp)]


class cascade_io(C.Structure):
    _fields_ = [("x", vp), ("key_gain", vp), ("x_out", vp), ("kept_tok", vp), ("kept_head", vp),
                ("tok_imp", vp), ("head_imp", vp), ("refetch_count", vp), ("sat_count", vp), ("dev_status", vp),
                ("caches", C.POINTER(decode_cache)), ("cap", i32), ("n_old", i32), ("dec_tok_imp", vp),
                ("trace_x", vp), ("trace_qkv", vp), ("trace_o", vp), ("trace_tok_imp", vp),
                ("trace_head_imp", vp), ("trace_flags", vp), ("attn_events", C.POINTER(vp))]


lib.spatten_abi_version.restype = i32
lib.spatten_status_string.restype = C.c_char_p
lib.spatten_status_string.argtypes = [i32]
lib.spatten_last_cuda_error.restype = C.c_char_p
lib.spatten_kernel_launch_count.restype = C.c_uint64
lib.spatten_set_wait_limit.restype = None
lib.spatten_set_wait_limit.argtypes = [C.c_uint32]
lib.spatten_quantize_kv.restype = i32
lib.spatten_quantize_kv.argtypes = [vp, i32, i32, i32, i32, i32, i64, vp, i64, vp, vp, vp, i32, i32, vp, vp, vp]
lib.spatten_attention_workspace_size.restype = sz
lib.spatten_attention_workspace_size.argtypes = [C.POINTER(attn_args)]
lib.spatten_attention_layer.restype = i32
lib.spatten_attention_layer.argtypes = [C.POINTER(attn_args), vp, sz, vp]
lib.spatten_attention_layer_noalloc.restype = i32
lib.spatten_attention_layer_noalloc.argtypes = [C.POINTER(attn_args), vp]
lib.spatten_selftest_exp2_poly.restype = i32
lib.spatten_selftest_exp2_poly.argtypes = [vp, vp, i64, vp]
lib.spatten_topk_workspace_size.restype = sz
lib.spatten_topk_workspace_size.argtypes = [i32, i32, i32]
lib.spatten_topk_select.restype = i32
lib.spatten_topk_select.argtypes = [vp, i32, i32, i64, i32, vp, i64, vp, i64, vp, vp, sz, vp, vp]
lib.spatten_gather_kept.restype = i32
lib.spatten_gather_kept.argtypes = [vp, i64, i64, i32, i64, i32, vp, i64, i32, vp, i64, i64, vp, i64, vp, i32, vp, vp]
lib.spatten_cascade_workspace_size.restype = sz
lib.spatten_cascade_workspace_size.argtypes = [C.POINTER(cascade_cfg)]
lib.spatten_cascade_forward.restype = i32
lib.spatten_cascade_forward.argtypes = [C.POINTER(cascade_cfg), C.POINTER(layer_weights), C.POINTER(cascade_io), vp, sz, vp]

# every extern "C" symbol of include/spatten.h
EXPORTS = ["spatten_abi_version", "spatten_status_string", "spatten_last_cuda_error",
           "spatten_kernel_launch_count", "spatten_quantize_kv",
           "spatten_attention_workspace_size", "spatten_attention_layer", "spatten_attention_layer_noalloc",
           "spatten_topk_workspace_size",
           "spatten_topk_select", "spatten_gather_kept", "spatten_cascade_workspace_size",
           "spatten_cascade_forward", "spatten_selftest_exp2_poly", "spatten_set_wait_limit"]


class SpattenError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.spatten_status_string(status).decode()
        if status == E_CUDA:
            msg += f" ({lib.spatten_last_cuda_error().decode()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != OK:
        raise SpattenError(status, where)


def ptr(t) -> int | None:
    """Device address of a torch tensor (None passes through; ints are taken as addresses)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- calls --------------------------------------------------------------------------------------
def quantize_kv(x, B, H, n, d_h, ld_tok, msb, lsb, cap, row0=0, scale_out=None, scale_in=None,
                row_gain=None, ld_gain=0, sat_count=None, dtype=None, stream=None):
    dt = dtype_code(x) if dtype is None and not isinstance(x, int) else dtype
    check(lib.spatten_quantize_kv(ptr(x), dt, B, H, n, d_h, ld_tok, ptr(row_gain), ld_gain, ptr(scale_in),
                                  ptr(msb), ptr(lsb), cap, row0, ptr(scale_out), ptr(sat_count), _stream(stream)),
          "spatten_quantize_kv")


def attention_workspace_size(args: attn_args) -> int:
    return lib.spatten_attention_workspace_size(C.byref(args))


def attention_layer(args: attn_args, ws, ws_bytes: int, stream=None):
    check(lib.spatten_attention_layer(C.byref(args), ptr(ws), ws_bytes, _stream(stream)), "spatten_attention_layer")


NOALLOC_SCRATCH_BYTES = 8 << 20   # SPATTEN_NOALLOC_SCRATCH_BYTES


def attention_layer_noalloc(args: attn_args, stream=None):
    """The attention layer without a caller workspace (library-owned scratch; see spatten.h)."""
    check(lib.spatten_attention_layer_noalloc(C.byref(args), _stream(stream)), "spatten_attention_layer_noalloc")


def topk_workspace_size(R: int, n: int, k: int) -> int:
    return lib.spatten_topk_workspace_size(R, n, k)


def topk_select(scores, R, n, ld, k, idx_out, ld_out, map=None, ld_map=0, comp_out=None, ws=None, ws_bytes=0,
                dev_status=None, stream=None):
    check(lib.spatten_topk_select(ptr(scores), R, n, ld, k, ptr(map), ld_map, ptr(idx_out), ld_out, ptr(comp_out),
                                  ptr(ws), ws_bytes, ptr(dev_status), _stream(stream)), "spatten_topk_select")


def gather_kept(src, src_batch, src_row, n_src, row_bytes, R, idx, ld_idx, k, dst, dst_batch, dst_row,
                compose_in=None, ld_compose=0, compose_out=None, check_index=0, dev_status=None, stream=None):
    check(lib.spatten_gather_kept(ptr(src), src_batch, src_row, n_src, row_bytes, R, ptr(idx), ld_idx, k, ptr(dst),
                                  dst_batch, dst_row, ptr(compose_in), ld_compose, ptr(compose_out), check_index,
                                  ptr(dev_status), _stream(stream)), "spatten_gather_kept")


def selftest_exp2_poly(x, y, n, stream=None):
    """y = 2^x by the attention kernels' FMA-pipe polynomial (diagnostic)."""
    check(lib.spatten_selftest_exp2_poly(ptr(x), ptr(y), n, _stream(stream)), "spatten_selftest_exp2_poly")


def kernel_launch_count() -> int:
    return int(lib.spatten_kernel_launch_count())


def set_wait_limit(polls: int) -> None:
    """Polls of one pipeline wait of the tensor-core kernels before they give up (0: default)."""
    lib.spatten_set_wait_limit(polls)


def cascade_workspace_size(cfg: cascade_cfg) -> int:
    return lib.spatten_cascade_workspace_size(C.byref(cfg))


def cascade_forward(cfg: cascade_cfg, weights, io: cascade_io, ws, ws_bytes: int, stream=None):
    """weights: sequence of (w_qkv, w_o) device tensors/pointers, one pair per layer."""
    arr = (layer_weights * cfg.L)(*[layer_weights(ptr(a), ptr(b)) for a, b in weights])
    check(lib.spatten_cascade_forward(C.byref(cfg), arr, C.byref(io), ptr(ws), ws_bytes, _stream(stream)),
          "spatten_cascade_forward")


def make_cfg(mode, B, T, D, H, d_h, L, dtype, token_keep, head_keep, quant, theta, sm_scale=0.0) -> cascade_cfg:
    c = cascade_cfg()
    c.mode, c.B, c.T, c.D, c.H, c.d_h, c.L, c.dtype = mode, B, T, D, H, d_h, L, dtype
    for l in range(L):
        c.token_keep[l] = token_keep[l]
        c.head_keep[l] = head_keep[l] if head_keep is not None else H
    c.quant, c.refetch_threshold, c.sm_scale = int(quant), float(theta), float(sm_scale)
    return c
