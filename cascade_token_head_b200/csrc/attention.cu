// spatten_attention_layer: argument checks, workspace layout and kernel choice.
//
//   tensor-core kernel (attn_tc.cu)   bf16 queries, quantized K/V, d_h in {64, 128}, many rows
//   decode kernel (attn_decode.cu)    one query row per (sequence, head), quantized K/V
//   CUDA-core kernel (attn_simt.cu)   everything else (the float32 configuration)
// Every kernel writes per-CTA partial importance sums to the workspace; attn_reduce adds them to
// tok_imp / head_imp in a fixed order.
#include <cmath>
#include <cstring>

#include "attention.cuh"

namespace spt {
namespace {

enum class Path { kSimt, kTc, kDecode };

// returns false when a forced kernel cannot run the problem
bool choose_path(const spatten_attn_args& a, Path* out) {
  switch (a.kernel) {
    case SPATTEN_ATTN_CUDA_CORE: *out = Path::kSimt; return true;
    case SPATTEN_ATTN_TENSOR_CORE: *out = Path::kTc; return attn_tc_supported(a);
    case SPATTEN_ATTN_DECODE:
    case SPATTEN_ATTN_DECODE_PREDICATED: *out = Path::kDecode; return attn_decode_supported(a);
    default: break;
  }
  if (attn_decode_supported(a)) *out = Path::kDecode;
  else if (attn_tc_supported(a)) *out = Path::kTc;
  else *out = Path::kSimt;
  return true;
}

int rows_per_cta(Path p) {
  switch (p) {
    case Path::kTc: return kTcRows;
    case Path::kDecode: return 1;
    default: return kSimtRows;
  }
}

int32_t validate(const spatten_attn_args& a) {
  if (a.B < 1 || a.H < 1 || a.n_q < 1 || a.n_kv < 1) return SPATTEN_E_ARG;
  if (a.B > 65535 || a.H > 1024) return SPATTEN_E_ARG;
  if (a.kernel < SPATTEN_ATTN_AUTO || a.kernel > SPATTEN_ATTN_DECODE_PREDICATED) return SPATTEN_E_ARG;
  if (a.v_keep < 0) return SPATTEN_E_ARG;
  if (a.d_h != 64 && a.d_h != 128) return SPATTEN_E_UNSUPPORTED;
  if (a.H_kept < 1 || a.H_kept > a.H) return SPATTEN_E_ARG;
  if (!a.head_idx && a.H_kept != a.H) return SPATTEN_E_ARG;
  if (a.head_idx && a.head_idx_ld != 0 && a.head_idx_ld < a.H_kept) return SPATTEN_E_SHAPE;
  if (!a.q || !a.o) return SPATTEN_E_ARG;
  if (a.q_dtype != SPATTEN_F32 && a.q_dtype != SPATTEN_BF16) return SPATTEN_E_ARG;
  const int64_t hd = static_cast<int64_t>(a.H) * a.d_h;
  if (a.q_ld_tok < hd || a.o_ld_tok < hd) return SPATTEN_E_SHAPE;
  if (a.quantized) {
    if (!a.k_msb || !a.k_lsb || !a.k_scale || !a.v_msb || !a.v_lsb || !a.v_scale) return SPATTEN_E_ARG;
    if (a.kv_cap < 1) return SPATTEN_E_ARG;
    if (!a.kv_idx && a.n_kv > a.kv_cap) return SPATTEN_E_SHAPE;
    if (a.kv_idx && a.kv_idx_ld < a.n_kv) return SPATTEN_E_SHAPE;
    if (!aligned16(a.k_msb) || !aligned16(a.v_msb) || !aligned16(a.k_lsb) || !aligned16(a.v_lsb))
      return SPATTEN_E_ALIGN;
  } else {
    if (!a.k || !a.v) return SPATTEN_E_ARG;
    if (a.kv_dtype != SPATTEN_F32 && a.kv_dtype != SPATTEN_BF16) return SPATTEN_E_ARG;
    if (a.kv_ld_tok < hd) return SPATTEN_E_SHAPE;
    if (a.kv_idx) return SPATTEN_E_UNSUPPORTED;
    if (a.n_kv != a.n_q) return SPATTEN_E_SHAPE;   // unquantized K/V share the query rows' layout
  }
  if (a.tok_imp && a.tok_imp_ld < (a.tok_imp_map ? 1 : a.n_kv)) return SPATTEN_E_SHAPE;
  if (a.tok_imp_map && a.tok_imp_map_ld < a.n_kv) return SPATTEN_E_SHAPE;
  if (a.refetch_flags && a.refetch_flags_ld != 0 && a.refetch_flags_ld < a.n_q) return SPATTEN_E_SHAPE;
  const int esz = a.q_dtype == SPATTEN_BF16 ? 2 : 4;
  if (!aligned16(a.q) || !aligned16(a.o) || (a.q_ld_tok * esz) % 16 != 0 || (a.o_ld_tok * esz) % 16 != 0)
    return SPATTEN_E_ALIGN;
  return SPATTEN_OK;
}

size_t layout(const spatten_attn_args& a, Path path, AttnProblem* p) {
  const int rows = rows_per_cta(path);
  const int64_t n_qt = ceil_div(a.n_q, rows);
  WsCursor c(p ? p->tok_part : nullptr, ~size_t(0));
  // per-CTA partials of the prefill kernels (the decode kernels keep per-item partials instead)
  const size_t parts = path == Path::kDecode ? 0 : static_cast<size_t>(a.B) * a.H_kept * n_qt;
  float* t = c.take<float>(parts * a.n_kv);
  float* h = c.take<float>(parts);
  int32_t* fl = nullptr;
  int32_t* fc = nullptr;
  float* fp = nullptr;
  float* fh = nullptr;
  const int64_t n_pair = ceil_div(a.n_q, 256);
  int items = 0;
  float* de = nullptr;
  float* ds = nullptr;
  float* dob = nullptr;
  int32_t* dfl = nullptr;
  if (path == Path::kDecode) {
    const int ir = decode_item_rows(a.d_h);
    items = static_cast<int>(ceil_div(a.n_kv, ir));
    const size_t bh = static_cast<size_t>(a.B) * a.H_kept;
    de = c.take<float>(2 * bh * a.n_kv);
    ds = c.take<float>(bh * items * 4);
    dob = c.take<float>(bh * items * 2 * a.d_h);
    if (a.kernel == SPATTEN_ATTN_DECODE_PREDICATED && a.refetch_threshold > 0.0f) dfl = c.take<int32_t>(bh);
  }
  if (path == Path::kTc) {
    fl = c.take<int32_t>(static_cast<size_t>(a.B) * a.H_kept * n_pair * 256);
    fc = c.take<int32_t>(static_cast<size_t>(a.B) * a.H_kept * n_pair);
    fp = c.take<float>(static_cast<size_t>(a.B) * a.H_kept * 2 * n_pair * a.n_kv);
    fh = c.take<float>(static_cast<size_t>(a.B) * a.H_kept * 2 * n_pair);
  }
  float* hc = nullptr;
  int32_t* vs = nullptr;
  uint8_t* vm = nullptr;
  if (value_pruning(a)) {
    const size_t bh = static_cast<size_t>(a.B) * a.H_kept;
    hc = c.take<float>(bh * a.n_kv);
    vs = c.take<int32_t>(bh * a.v_keep);
    if (path != Path::kDecode) vm = c.take<uint8_t>(bh * a.n_kv);
  }
  if (p) {
    p->head_col = hc;
    p->v_sel = vs;
    p->v_mask = vm;
    p->qt_rows = rows;
    p->n_qt = static_cast<int>(n_qt);
    p->tok_part = t;
    p->head_part = h;
    p->n_pair = static_cast<int>(n_pair);
    p->flag_list = fl;
    p->flag_cnt = fc;
    p->full_part = fp;
    p->full_head = fh;
    p->dec_items = items;
    p->dec_e = de;
    p->dec_stat = ds;
    p->dec_o = dob;
    p->dec_flag = dfl;
  }
  return c.used;
}

}  // namespace
}  // namespace spt

extern "C" size_t spatten_attention_workspace_size(const spatten_attn_args* a) {
  using namespace spt;
  Path path;
  if (!a || validate(*a) != SPATTEN_OK || !choose_path(*a, &path)) return 0;
  return layout(*a, path, nullptr);
}

namespace spt {
int32_t attention_layer_timed(const spatten_attn_args* args, void* ws, size_t ws_bytes, cudaStream_t st,
                              cudaEvent_t ev_begin, cudaEvent_t ev_end) {
  if (!args) return SPATTEN_E_ARG;
  SPT_TRY(validate(*args));
  AttnProblem p;
  std::memcpy(&p.a, args, sizeof(spatten_attn_args));
  p.wait_limit = wait_limit_setting();
  if (!(p.a.sm_scale > 0.0f)) p.a.sm_scale = 1.0f / std::sqrt(static_cast<float>(p.a.d_h));
  if (p.a.head_idx_ld == 0) p.a.head_idx_ld = p.a.H_kept;
  if (p.a.refetch_flags_ld == 0) p.a.refetch_flags_ld = p.a.n_q;
  Path path;
  if (!choose_path(p.a, &path)) return SPATTEN_E_UNSUPPORTED;
  p.tok_part = static_cast<float*>(ws);
  const size_t need = layout(p.a, path, &p);
  if (!ws || ws_bytes < need) return SPATTEN_E_WORKSPACE;
  // inside a stream capture, external records become timing event nodes of the graph
  unsigned ev_flags = 0;
  if (ev_begin || ev_end) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    SPT_CUDA(cudaStreamIsCapturing(st, &cs));
    if (cs == cudaStreamCaptureStatusActive) ev_flags = cudaEventRecordExternal;
  }
  if (ev_begin) SPT_CUDA(cudaEventRecordWithFlags(ev_begin, st, ev_flags));
  auto run = [&](const AttnProblem& q) -> int32_t {
    switch (path) {
      case Path::kTc: return attn_tc_launch(q, st);
      case Path::kDecode: return attn_decode_launch(q, st);   // its own combine step reduces
      default: return attn_simt_launch(q, st);
    }
  };
  if (!value_pruning(p.a)) {
    SPT_TRY(run(p));
    if (path != Path::kDecode && (p.a.tok_imp || p.a.head_imp)) SPT_TRY(attn_reduce_launch(p, st));
  } else {
    // local value pruning: each head's column sums of P select the V vectors it keeps
    const int32_t R = p.a.B * p.a.H_kept;
    if (path == Path::kDecode) {
      // items and combine: token importance and each head's probabilities (p.head_col); the
      // outputs are left to the pruned-output kernel (p.v_sel set)
      SPT_TRY(run(p));
      SPT_TRY(spatten_topk_select(p.head_col, R, p.a.n_kv, p.a.n_kv, p.a.v_keep, nullptr, 0, p.v_sel, p.a.v_keep,
                                  nullptr, nullptr, 0, p.a.dev_status, st));
      SPT_TRY(attn_decode_pruned_out_launch(p, st));
    } else {
      // run 1: token importance, refetch flags and counts, per-head column sums
      AttnProblem r1 = p;
      r1.a.head_imp = nullptr;
      r1.v_mask = nullptr;
      SPT_TRY(run(r1));
      if (r1.a.tok_imp) SPT_TRY(attn_reduce_launch(r1, st));
      SPT_TRY(attn_head_colsum_launch(r1, st));
      SPT_TRY(spatten_topk_select(p.head_col, R, p.a.n_kv, p.a.n_kv, p.a.v_keep, nullptr, 0, p.v_sel, p.a.v_keep,
                                  nullptr, nullptr, 0, p.a.dev_status, st));
      uint8_t* mask = const_cast<uint8_t*>(p.v_mask);
      SPT_TRY(attn_value_mask_launch(p, mask, st));
      // run 2: the same layer with the dropped V vectors masked: outputs and head importance
      AttnProblem r2 = p;
      r2.a.tok_imp = nullptr;
      r2.a.refetch_flags = nullptr;
      r2.a.refetch_count = nullptr;
      SPT_TRY(run(r2));
      if (r2.a.head_imp) SPT_TRY(attn_reduce_launch(r2, st));
    }
  }
  if (ev_end) SPT_CUDA(cudaEventRecordWithFlags(ev_end, st, ev_flags));
  return SPATTEN_OK;
}
}  // namespace spt

extern "C" int32_t spatten_attention_layer(const spatten_attn_args* args, void* ws,
                                           size_t ws_bytes, void* stream) {
  spt::AbiRange nvtx_range("spatten_attention_layer");
  return spt::attention_layer_timed(args, ws, ws_bytes, spt::as_stream(stream), nullptr, nullptr);
}
