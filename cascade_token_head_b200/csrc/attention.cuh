// Internal interface between the attention dispatcher and its kernels.
#pragma once

#include "common.cuh"

namespace spt {

// Resolved attention problem (validated by the dispatcher).
constexpr uint32_t kDefaultWaitLimit = 1u << 26;   // about a second of polling on one mbarrier phase
// the limit given to the kernels of the next calls (spatten_set_wait_limit; 0 = the default)
uint32_t wait_limit_setting();

struct AttnProblem {
  spatten_attn_args a;       // copy of the caller's arguments, sm_scale resolved
  int qt_rows;               // query rows per CTA of the chosen kernel
  int n_qt;                  // query tiles = ceil(n_q / qt_rows)
  float* tok_part;           // ws [B][H_kept][n_qt][n_kv] per-CTA column sums of P
  float* head_part;          // ws [B][H_kept][n_qt] per-CTA sum |O|
  // tensor-core path only: query rows flagged for refetch are recomputed at full precision by a
  // second kernel, in packed 128-row tiles of the flagged rows of each 256-row query pair tile
  int n_pair;                // ceil(n_q / 256)
  int32_t* flag_list;        // ws [B][H_kept][n_pair][256] flagged row ids, ascending
  int32_t* flag_cnt;         // ws [B][H_kept][n_pair] number of flagged rows
  float* full_part;          // ws [B][H_kept][2*n_pair][n_kv] column sums of the packed tiles
  float* full_head;          // ws [B][H_kept][2*n_pair] sum |O| of the packed tiles
  // decode path only: per-item partials of the streaming kernel (an item is a run of
  // decode_item_rows(d_h) consecutive entries of a row's key list)
  int dec_items;             // items per (b, kept head) = ceil(n_kv / item rows)
  float* dec_e;              // ws [2][B][H_kept][n_kv] exp(s - item max): MSB-only, full precision
  float* dec_stat;           // ws [B][H_kept][dec_items][4] item max and sum, both variants
  float* dec_o;              // ws [B][H_kept][dec_items][2][d_h] item sum of exp * V, both variants
  int32_t* dec_flag = nullptr;  // ws [B][H_kept] predicated form only: rows whose LSBs are read
  // local value pruning (a.v_keep in [1, n_kv)): each kept head's column sums of P, its kept keys
  // and (prefill) the V mask of the second run
  float* head_col = nullptr;        // ws [B][H_kept][n_kv] (decode: written by the combine step)
  int32_t* v_sel = nullptr;         // ws [B][H_kept][v_keep] kept keys, ascending; decode: set when
                                    // the combine step leaves the outputs to the pruned-output kernel
  const uint8_t* v_mask = nullptr;  // ws [B][H_kept][n_kv] 1 = V vector kept (prefill second run)
  // tensor-core kernels: polls of one pipeline wait before the kernel gives up (SPATTEN_E_TIMEOUT)
  uint32_t wait_limit = kDefaultWaitLimit;
};

// Kernels (each returns a status after launching on `st`).
int32_t attn_simt_launch(const AttnProblem& p, cudaStream_t st);
int32_t attn_tc_launch(const AttnProblem& p, cudaStream_t st);
int32_t attn_decode_launch(const AttnProblem& p, cudaStream_t st);
bool attn_tc_supported(const spatten_attn_args& a);
bool attn_decode_supported(const spatten_attn_args& a);
int decode_item_rows(int d_h);    // keys per item of the decode kernel
constexpr int kTcRows = 128;      // query rows per CTA of the tensor-core kernel
constexpr int kSimtRows = 32;     // query rows per CTA of the CUDA-core kernel

// spatten_attention_layer with optional events recorded around all of its kernels (attention, the
// pruned-head zero fill, the refetch pass and the importance reduction).
int32_t attention_layer_timed(const spatten_attn_args* a, void* ws, size_t ws_bytes, cudaStream_t st,
                              cudaEvent_t ev_begin, cudaEvent_t ev_end);

// K and V of one projection buffer quantized in one launch (quantize.cu)
int32_t quantize_kv_pair(const void* k, const void* v, int32_t dtype, int32_t B, int32_t H, int32_t n, int32_t d_h,
                         int64_t ld_tok, const float* k_gain, int64_t ld_gain, const float* k_scale_in,
                         const float* v_scale_in, int8_t* k_msb, uint8_t* k_lsb, int8_t* v_msb, uint8_t* v_lsb,
                         int32_t cap, int32_t row0, float* k_scale_out, float* v_scale_out, int32_t* sat_count,
                         cudaStream_t st);

// Fixed-order reduction of the per-CTA partials into tok_imp / head_imp.
int32_t attn_reduce_launch(const AttnProblem& p, cudaStream_t st);
// Local value pruning, prefill: per-head column sums of the partials (same order as the reduction)
// into p.head_col; the V mask from the kept key lists p.v_sel
int32_t attn_head_colsum_launch(const AttnProblem& p, cudaStream_t st);
int32_t attn_value_mask_launch(const AttnProblem& p, uint8_t* mask, cudaStream_t st);
// Local value pruning, decode: O = sum over the kept keys of P_j v_j, head importance, flags
int32_t attn_decode_pruned_out_launch(const AttnProblem& p, cudaStream_t st);
inline bool value_pruning(const spatten_attn_args& a) { return a.v_keep > 0 && a.v_keep < a.n_kv; }

// Head slot -> original head id; slots >= H_kept name the pruned heads in ascending order.
__device__ __forceinline__ int head_of_slot(const spatten_attn_args& a, int b, int slot) {
  if (!a.head_idx) return slot;
  const int32_t* hi = a.head_idx + static_cast<int64_t>(b) * a.head_idx_ld;
  if (slot < a.H_kept) return hi[slot];
  int want = slot - a.H_kept, seen = 0;
  for (int h = 0; h < a.H; ++h) {
    bool kept = false;
    for (int s = 0; s < a.H_kept; ++s) kept |= (hi[s] == h);
    if (!kept) {
      if (seen == want) return h;
      ++seen;
    }
  }
  return -1;
}

}  // namespace spt
