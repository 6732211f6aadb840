/*
 * spatten.h -- C ABI of libspatten.so: SpAtten-style cascade token/head pruning with
 * progressive (MSB + LSB) K/V quantization, for one NVIDIA B200 (sm_100a).
 *
 * Source of the method: "SpAtten: Efficient Sparse Attention Architecture with Cascade Token and
 * Head Pruning" (Wang, Zhang, Han; arXiv 2012.09852v3), as summarised on its paperlayer.ai page.
 * Section names below are that page's.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Ownership: the caller owns every buffer.  Pointers named as "device" must be device
 *    memory of the current CUDA device; the library allocates no device memory.  Calls that need
 *    scratch take (ws, ws_bytes); the matching *_workspace_size() query returns the size needed.
 *  - Streams: every call is asynchronous on the given stream (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream) and returns after enqueueing its kernels.
 *  - Errors: every call returns an int32 status (spatten_status below) and never aborts or
 *    throws.  Host-side argument checks run before any launch; a failing call enqueues nothing.
 *    Errors found on the device (an out-of-range index in checked mode, a bounded wait that gave
 *    up) are written to an optional device int32 `dev_status` (first error wins, 0 = OK); read it
 *    after synchronising.  spatten_status_string() names a status; after SPATTEN_E_CUDA,
 *    spatten_last_cuda_error() returns the CUDA error string of the calling thread.
 *  - Importance buffers are accumulated with += and never cleared by the per-kernel calls;
 *    spatten_cascade_forward() zeroes its own at the start of a prefill pass.
 *  - Dense tensors are row-major.  Element (b, h, t, d) of a projection tensor with heads packed
 *    in a token row is at  base[(b * n + t) * ld_tok + h * d_h + d]  (ld_tok in elements).
 *  - K/V planes (the progressive-quantization storage, §III.A "Progressive Quantization" and
 *    §IV "Quantization Support"): per (b, h) `cap` rows of d_h codes.
 *      MSB plane  int8   [B][H][cap][d_h]      q >> 4 (arithmetic shift, -128..127)
 *      LSB plane  uint8  [B][H][cap][d_h / 2]  q & 15, element 2c in bits 0-3, 2c+1 in bits 4-7
 *      scale      float  [B][H]                one float32 scale per (sequence, head, tensor)
 *    with the 12-bit code q in [-2047, 2047] and the value x ~= scale * q = scale*(16*MSB + LSB).
 *    An MSB-only read zero-fills the LSB field: x_msb = scale * 16 * MSB.
 */
#ifndef SPATTEN_H
#define SPATTEN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPATTEN_ABI_VERSION 1

/* ---- status codes ---------------------------------------------------------------------- */
enum spatten_status {
  SPATTEN_OK = 0,
  SPATTEN_E_ARG = 1,         /* null pointer or out-of-range scalar argument              */
  SPATTEN_E_SHAPE = 2,       /* inconsistent sizes (k > n, ld < row length, ...)          */
  SPATTEN_E_ALIGN = 3,       /* a pointer or stride breaks the 16-byte alignment rule      */
  SPATTEN_E_WORKSPACE = 4,   /* ws is NULL or ws_bytes is below *_workspace_size()         */
  SPATTEN_E_NONFINITE = 5,   /* NaN input found (top-k scores)                             */
  SPATTEN_E_CUDA = 6,        /* a CUDA launch or runtime call failed                       */
  SPATTEN_E_TIMEOUT = 7,     /* a bounded device-side wait gave up                         */
  SPATTEN_E_UNSUPPORTED = 8, /* valid but not implemented (e.g. d_h not in {64, 128})      */
  SPATTEN_E_INDEX = 9,       /* (device) an index list entry was outside [0, n)            */
  SPATTEN_E_RANGE = 10       /* (device) a value left the range of the kernel's operand type:
                                a bf16 query of magnitude 65536 or more (the smallest bf16
                                value past fp16's 65504), infinite or NaN, given to the
                                tensor-core kernels, which take fp16 operands; it is stored
                                saturated to +-65504 and the call's results are unreliable     */
};

/* ---- element types ------------------------------------------------------------------------ */
enum spatten_dtype { SPATTEN_F32 = 0, SPATTEN_BF16 = 1 };

int32_t spatten_abi_version(void);
const char* spatten_status_string(int32_t status);
const char* spatten_last_cuda_error(void);
/* Number of kernels this library has launched in this process (its own kernels only; the cuBLASLt
 * projections are not counted).  A diagnostic for benchmarks and tests. */
uint64_t spatten_kernel_launch_count(void);
/* Polls of one pipeline wait (an mbarrier phase) after which the tensor-core attention kernels of
 * the calls that follow give up: the kernel stops its work, waits (with a bound of its own) for the
 * copies and MMAs it already started, releases its tensor memory, returns, and the call reports
 * SPATTEN_E_TIMEOUT in its dev_status word.  0 restores the default (2^26 polls, about a second).
 * Process-wide; read when a call is launched (a CUDA graph keeps the value it was captured with).
 * A diagnostic: a small value makes the waits run out on purpose, so that the timeout path can be
 * checked without a fault. */
void spatten_set_wait_limit(uint32_t polls);

/* =============================================================================================
 * spatten_quantize_kv -- progressive 12-bit quantization of K or V into an MSB and an LSB plane
 * (§III.A "Progressive Quantization": MSBs are fetched first, LSBs only on low confidence;
 *  §IV "Quantization Support": the bitwidth converter splits and concatenates MSBs and LSBs).
 *
 *  x         device, dtype elements; x(b,h,t,d) = x[(b*n + t)*ld_tok + h*d_h + d], t < n.
 *  row_gain  device float [B][ld_gain] or NULL; x is multiplied by row_gain[b*ld_gain + t]
 *            (in float32) before quantization (used for boosted keys).
 *  scale_in  device float [B*H] or NULL.  NULL: the scale of each (b, h) block is
 *            amax_{t,d} |x| / 2047 in float32 (1 if amax == 0) and is written to scale_out.
 *            Non-NULL: that scale is used (decode append with the prompt-time scale); codes
 *            saturate at +-2047 and the number of saturated elements is added to *sat_count.
 *  msb, lsb  device planes with `cap` rows per (b, h); rows [row0, row0 + n) are written.
 *  scale_out device float [B*H]; required when scale_in is NULL, else ignored (may be NULL).
 *  sat_count device int32 (optional, +=).
 *  Codes: q = clamp(rint_half_even(float32(x) / s), -2047, 2047) with an IEEE float32 divide.
 *  Requirements: d_h even and a multiple of 8, 1 <= n, row0 + n <= cap, B, H >= 1.
 * ============================================================================================= */
int32_t spatten_quantize_kv(const void* x, int32_t dtype, int32_t B, int32_t H, int32_t n,
                            int32_t d_h, int64_t ld_tok, const float* row_gain, int64_t ld_gain,
                            const float* scale_in, int8_t* msb, uint8_t* lsb, int32_t cap,
                            int32_t row0, float* scale_out, int32_t* sat_count, void* stream);

/* =============================================================================================
 * spatten_attention_layer -- one attention layer over the kept tokens and heads, returning the
 * outputs plus the token- and head-importance increments (§II "Attention mechanism", §II
 * "Cascade pruning", §II.B "Token pruning", §IV.E "Progressive Quantization").
 *
 * For every sequence b and kept head h = head_idx[b][s] (s < H_kept), query row i < n_q:
 *   S_ij  = sm_scale * q_i . k_j over the key list j < n_kv (through kv_idx when given)
 *   MSB pass (quantized K/V): k_j = k_scale*16*MSB_j; ell_i = sum_j exp(S_ij - max_j S_ij).
 *   Refetch: if 1/ell_i < refetch_threshold (strict), row i is recomputed with the full 12-bit
 *   K and V (LSB plane read); theta <= 0 never refetches, theta > 1 always does.
 *   P_i = softmax(S_i) (final precision), O_i = sum_j P_ij v_j (v_j at the row's precision).
 *   tok_imp[b][map(j)] += sum_{kept h, i} P_ij       (map(j) = tok_imp_map[b][j] or j)
 *   head_imp[b][h]     += sum_{i,d} |O_id|
 * Importance sums are reduced in a fixed order (reruns are bit-identical).
 *
 * Local value pruning (§III.A "Local Value Pruning": after the softmax a head discards its
 * low-probability V vectors, for that head only), when 1 <= v_keep < n_kv: head h keeps the V
 * vectors of the v_keep keys ranked first by (larger c_hj = sum_i P_ij, the key's column sum of the
 * head's final probabilities, then lower j); its output becomes O_i = sum_{j kept} P_ij v_j with no
 * renormalisation, and head_imp uses that output.  The token importance and the refetch decisions
 * are those of the full probabilities.  The layer then runs its attention twice (once for the
 * column sums, once with the V mask) and needs the larger workspace the size query reports.
 * ============================================================================================= */
typedef struct spatten_attn_args {
  int32_t B, H;              /* sequences, heads in the layer (original head count)          */
  int32_t n_q, n_kv, d_h;    /* query rows, key rows, head dim (64 or 128)                   */
  int32_t H_kept;            /* kept heads per sequence (1..H)                               */
  const int32_t* head_idx;   /* device [B][head_idx_ld] ascending original head ids of the    */
  int64_t head_idx_ld;       /* H_kept kept heads (NULL = all heads 0..H-1); ld 0 = H_kept   */

  const void* q;             /* device, q_dtype; q(b,h,i,d) = q[(b*n_q + i)*q_ld_tok + h*d_h + d] */
  int32_t q_dtype;
  int64_t q_ld_tok;

  int32_t quantized;         /* 1: K/V come from the planes below; 0: from k/v (no refetch)  */
  const int8_t* k_msb;       /* device planes, kv_cap rows per (b, h)                        */
  const uint8_t* k_lsb;
  const float* k_scale;      /* device [B*H]                                                 */
  const int8_t* v_msb;
  const uint8_t* v_lsb;
  const float* v_scale;
  int32_t kv_cap;

  const void* k;             /* quantized == 0: device, kv_dtype, like q with n_kv rows      */
  const void* v;
  int32_t kv_dtype;
  int64_t kv_ld_tok;

  const int32_t* kv_idx;     /* device [B][kv_idx_ld] plane/row ids of the n_kv keys, or NULL  */
  int64_t kv_idx_ld;

  float sm_scale;            /* <= 0 selects 1/sqrt(d_h)                                     */
  float refetch_threshold;   /* theta                                                        */

  void* o;                   /* device, q_dtype; o(b,h,i,d) = o[(b*n_q + i)*o_ld_tok + h*d_h + d] */
  int64_t o_ld_tok;
  int32_t zero_pruned_heads; /* 1: write zeros to o for the H - H_kept pruned heads          */

  float* tok_imp;            /* device [B][tok_imp_ld] (+=) or NULL                          */
  int64_t tok_imp_ld;
  const int32_t* tok_imp_map;/* device [B][tok_imp_map_ld] or NULL (identity)                */
  int64_t tok_imp_map_ld;
  float* head_imp;           /* device [B][H] (+=) or NULL                                   */

  uint8_t* refetch_flags;    /* device [B][H][refetch_flags_ld] (kept heads written) or NULL  */
  int64_t refetch_flags_ld;  /* row stride of refetch_flags; 0 = n_q                          */
  int32_t* refetch_count;    /* device int32 (+= number of refetched rows) or NULL           */
  int32_t* dev_status;       /* device int32 or NULL                                         */
  int32_t kernel;            /* spatten_attn_kernel: 0 = choose automatically                */
  int32_t v_keep;            /* local value pruning: 0 (or >= n_kv) keeps every V vector;     */
                             /* else each kept head keeps v_keep of them (see below)          */
} spatten_attn_args;

/* Kernel choice for spatten_attention_layer.  AUTO picks the tensor-core kernel for bf16
 * queries over quantized K/V, the decode kernel for one query row per (sequence, head), and the
 * CUDA-core kernel otherwise; CUDA_CORE forces the float32 CUDA-core kernel (a cross-check of
 * the other two on the same inputs).  A forced kernel that cannot run the problem returns
 * SPATTEN_E_UNSUPPORTED. */
enum spatten_attn_kernel {
  SPATTEN_ATTN_AUTO = 0,
  SPATTEN_ATTN_CUDA_CORE = 1,
  SPATTEN_ATTN_TENSOR_CORE = 2,
  SPATTEN_ATTN_DECODE = 3,
  /* the decode kernel with a predicated LSB fetch (theta > 0): a first pass over the MSB planes of
   * every row, the refetch decision per row, then a full-precision pass that reads the LSB planes
   * of the flagged rows only (their MSB planes again, usually from L2).  The results are the
   * same, bit for bit, as SPATTEN_ATTN_DECODE's; it reads fewer bytes when few rows refetch and
   * costs a second pass when most do. */
  SPATTEN_ATTN_DECODE_PREDICATED = 4
};

size_t spatten_attention_workspace_size(const spatten_attn_args* a);
int32_t spatten_attention_layer(const spatten_attn_args* a, void* ws, size_t ws_bytes,
                                void* stream);

/* ---------------------------------------------------------------------------------------------
 * spatten_attention_layer_noalloc -- spatten_attention_layer for callers that cannot allocate.
 * (The paper has no counterpart: this is a deployment convenience of this library.)
 *
 * Some callers have no way to allocate device memory at all -- a plugin whose host application
 * owns every allocation, a real-time loop that must never enter the CUDA allocator, code that is
 * only handed its input and output buffers -- and so cannot supply the workspace the call above
 * needs.  This entry point takes the same arguments without (ws, ws_bytes): its scratch lives in
 * a fixed array of SPATTEN_NOALLOC_SCRATCH_BYTES in device global memory owned by the library,
 * which every GPU that loads the library holds until the process exits.  It calls no
 * cudaMalloc/cudaFree and no allocating library routine.
 *  - Limit: problems whose spatten_attention_workspace_size() exceeds the array are rejected with
 *    SPATTEN_E_WORKSPACE before anything is launched (use the workspace entry point for them).
 *  - Set-up: the first call on each device (with that device current) looks up the array's
 *    device address with cudaGetSymbolAddress and caches it; make that first call before any
 *    stream capture.
 *  - Sharing: all calls use the same array, so calls that overlap on the GPU (other streams or
 *    threads) race on it; serialise them.  Everything a call reads from the array it has written
 *    itself first, so no clearing is needed between calls.
 * The caller still passes every input and output buffer in `a`, as for the call above.
 * --------------------------------------------------------------------------------------------- */
#define SPATTEN_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
int32_t spatten_attention_layer_noalloc(const spatten_attn_args* a, void* stream);

/* =============================================================================================
 * spatten_topk_select -- per row, the k indices with the largest scores, ranked by (higher
 * score, then lower index), written in ascending order (§II "Cascade pruning": keep the top-k
 * tokens by the pruning ratio; §IV.B "Top-k Engine": find the k-th largest value as a threshold,
 * filter, then eliminate the gaps).  -0.0 and +0.0 are equal; NaN gives SPATTEN_E_NONFINITE in
 * dev_status and an unspecified selection.
 *
 *  scores   device float; row r element j is scores[r*ld + (map ? map[r*ld_map + j] : j)].
 *  map      device int32 [R][ld_map] or NULL: reads scores through an index list (gather fused).
 *  idx_out  device int32 [R][ld_out] or NULL: positions j (0 <= j < n) of the selected
 *           elements.  May be NULL only when comp_out is given.
 *  comp_out device int32 [R][ld_out] or NULL: map[r][idx_out[r][c]] (index-map composition);
 *           requires map.
 *  Requirements: R >= 1, 1 <= n, 0 <= k <= n, ld >= n when map is NULL, ld_out >= k.
 *  Workspace (ws, ws_bytes): optional, device memory of spatten_topk_workspace_size(R, n, k)
 *  bytes (0 for rows shorter than 65,536 keys).  Given it, rows of at least 65,536 keys read
 *  directly (map NULL, scores 16-byte aligned, ld a multiple of 4) take a one-read streaming path:
 *  a 16 K-key sample (8 K below 512 K keys) brackets the k-th key, one pass over the scores marks
 *  the keys above the bracket in a bit mask and collects the bracket's keys, the exact threshold is
 *  chosen among them, and the output is written from the mask and the selected bracket keys; rows
 *  whose bracket misses fall back to the cluster radix select.  Without it (or with fewer bytes)
 *  every row takes the cluster radix select.  Results are identical either way.  The workspace
 *  holds only this call's intermediates (nothing to clear): later calls on the same stream may
 *  reuse it, calls that overlap on the GPU need one each.
 * ============================================================================================= */
size_t spatten_topk_workspace_size(int32_t R, int32_t n, int32_t k);
int32_t spatten_topk_select(const float* scores, int32_t R, int32_t n, int64_t ld, int32_t k,
                            const int32_t* map, int64_t ld_map, int32_t* idx_out, int64_t ld_out,
                            int32_t* comp_out, void* ws, size_t ws_bytes, int32_t* dev_status,
                            void* stream);

/* =============================================================================================
 * spatten_gather_kept -- drop pruned rows: copy the kept rows of each batch into a compact
 * buffer (§III.A "Cascade Token Pruning": a pruned token's Q, K and V leave all following
 * layers; §IV.B "Zero Elimination"; §IV "Architecture Overview": pruning makes row access random).
 *
 *  For r < R, j < k:  dst[r*dst_batch + j*dst_row] <- src[r*src_batch + idx[r*ld_idx + j]*src_row]
 *  copying row_bytes bytes (strides in bytes).  If compose_in and compose_out are given:
 *  compose_out[r*ld_idx + j] = compose_in[r*ld_compose + idx[r*ld_idx + j]].
 *  Requirements: row_bytes a multiple of 4; 16-byte vector copies are used when src, dst,
 *  strides and row_bytes are all multiples of 16.  With check_index != 0 an index outside
 *  [0, n_src) is skipped and reported as SPATTEN_E_INDEX in dev_status.
 * ============================================================================================= */
int32_t spatten_gather_kept(const void* src, int64_t src_batch, int64_t src_row, int32_t n_src,
                            int64_t row_bytes, int32_t R, const int32_t* idx, int64_t ld_idx,
                            int32_t k, void* dst, int64_t dst_batch, int64_t dst_row,
                            const int32_t* compose_in, int64_t ld_compose, int32_t* compose_out,
                            int32_t check_index, int32_t* dev_status, void* stream);

/* =============================================================================================
 * spatten_cascade_forward -- L attention-only layers with cascade token and head pruning
 * (§II "Cascade pruning", §III.A "Cascade Token Pruning" / "Cascade Head Pruning").
 *
 * PREFILL (summarization): for layer l with the k_l kept tokens S_l and H_l kept heads of every
 * sequence:  [Q|K|V] = X_S @ W_qkv[l] (all heads, cuBLASLt), K rows times key_gain, K/V
 * quantized per (b, head) when quant != 0, attention with importance, X_S += O @ W_o[l] (pruned
 * heads give 0; the fully-connected layers run on the library GEMM, as the paper runs them off
 * the attention engine, §II.B "Motivation").  Then S_{l+1} = top-k_{l+1} of the cumulative token
 * importance over S_l and the H_{l+1} heads with the largest cumulative head importance.
 *
 * DECODE_STEP (generation, §II "Attention-based NLP models"): one new token per sequence.  Per
 * layer: project x_l; append its K/V to the layer's cache planes at row n (prompt-time scale,
 * saturating); attend over S_l (S_0 = rows 0..n); I += P; x_{l+1} = x_l + O @ W_o;
 * S_{l+1} = top-k_{l+1}(I restricted to S_l) with k_l = token_keep[l] (all heads kept).
 *
 * STREAMS: all work is ordered on `stream`.  The next layer's selections run on a second stream
 * of the library's own (one per device and host thread, created on the first call made outside a
 * stream capture), forked from `stream` after the attention step and joined back by events before
 * their results are read, so that they overlap the projections; a stream capture of the call
 * captures both.  A call made inside a capture before that stream exists runs them on `stream`.
 * ============================================================================================= */
enum spatten_mode { SPATTEN_PREFILL = 0, SPATTEN_DECODE_STEP = 1 };

#define SPATTEN_MAX_LAYERS 64

typedef struct spatten_cascade_cfg {
  int32_t mode;              /* spatten_mode                                                 */
  int32_t B, T, D, H, d_h, L;/* T: tokens (PREFILL) or cache rows n+1 after the append (DECODE) */
  int32_t dtype;             /* activations/weights: SPATTEN_F32 or SPATTEN_BF16             */
  int32_t token_keep[SPATTEN_MAX_LAYERS]; /* k_l entering layer l; token_keep[0] == T          */
  int32_t head_keep[SPATTEN_MAX_LAYERS];  /* H_l; head_keep[0] == H (PREFILL; DECODE: all H)   */
  int32_t quant;             /* 1: progressive K/V quantization (required for DECODE_STEP)    */
  float refetch_threshold;   /* theta                                                        */
  float sm_scale;            /* <= 0 selects 1/sqrt(d_h)                                     */
} spatten_cascade_cfg;

typedef struct spatten_layer_weights {
  const void* w_qkv;         /* device [D][3*H*d_h] row-major: [W_q | W_k | W_v], dtype      */
  const void* w_o;           /* device [H*d_h][D] row-major, dtype                            */
} spatten_layer_weights;

typedef struct spatten_decode_cache {
  int8_t* k_msb; uint8_t* k_lsb; const float* k_scale; /* planes [B][H][cap][..], scale [B*H]   */
  int8_t* v_msb; uint8_t* v_lsb; const float* v_scale;
} spatten_decode_cache;

typedef struct spatten_cascade_io {
  /* PREFILL */
  const void* x;             /* device [B][T][D] dtype, input hidden states (not modified)   */
  const float* key_gain;     /* device [B][T] or NULL: K-row factor after projection          */
  void* x_out;               /* device [B][token_keep[L-1]][D]: final rows of S_{L-1}         */
  int32_t* kept_tok;         /* device [L][B][T]: S_l in row l (first k_l entries, ascending) */
  int32_t* kept_head;        /* device [L][B][H]: kept heads of layer l (first H_l, ascending)*/
  float* tok_imp;            /* device [B][T]: cumulative token importance (zeroed at start)   */
  float* head_imp;           /* device [B][H]: cumulative head importance (zeroed at start)    */
  int32_t* refetch_count;    /* device [L]: refetched query rows per layer (zeroed at start)   */
  int32_t* sat_count;        /* device int32 (+=) or NULL: saturated codes on decode append    */
  int32_t* dev_status;       /* device int32 or NULL                                          */
  /* DECODE_STEP (x and x_out are [B][D]; kept_tok is [L][B][cap]; the traces drop the T axis:
   * trace_x [L][B][D], trace_qkv [L][B][3*H*d_h], trace_o [L][B][H*d_h], trace_flags [L][B][H]) */
  const spatten_decode_cache* caches; /* host array of L device caches                         */
  int32_t cap;               /* rows per (b, h) in the cache planes                            */
  int32_t n_old;             /* rows already in the caches (the new token goes to row n_old)   */
  float* dec_tok_imp;        /* device [B][cap]: cumulative importance, persists across steps  */
  /* optional per-layer trace for layer-by-layer checks (device, NULL = off)                    */
  void* trace_x;             /* [L][B][T][D]   X entering layer l (compact rows, first k_l)   */
  void* trace_qkv;           /* [L][B][T][3*H*d_h] projections of layer l                      */
  void* trace_o;             /* [L][B][T][H*d_h]   attention outputs of layer l                */
  float* trace_tok_imp;      /* [L][B][T] (PREFILL) / [L][B][cap] (DECODE): I after layer l    */
  float* trace_head_imp;     /* [L][B][H]  J after layer l                                     */
  uint8_t* trace_flags;      /* [L][B][H][T] refetch flags of layer l                          */
  /* optional timing hook: host array of 2*L cudaEvent_t (as void*); event 2l is recorded on the
   * stream right before layer l's attention kernels and event 2l+1 right after them (after the
   * importance reduction), so callers can time step a2/a3 of each layer alone.  NULL = off.    */
  void* const* attn_events;
} spatten_cascade_io;

size_t spatten_cascade_workspace_size(const spatten_cascade_cfg* cfg);
int32_t spatten_cascade_forward(const spatten_cascade_cfg* cfg, const spatten_layer_weights* w,
                                spatten_cascade_io* io, void* ws, size_t ws_bytes, void* stream);

/* =============================================================================================
 * Diagnostics
 *
 * spatten_selftest_exp2_poly -- y[i] = 2^x[i] by the polynomial the tensor-core attention kernels
 * use for a share of their softmax exponentials (Cody-Waite reduction to [-1/2, 1/2] and a
 * degree-5 minimax polynomial; §IV.E "Softmax" only says exponentials are computed).  Defined for
 * x <= 0, the range of softmax exponents; x < -126 gives 2^-126.  Maximum relative error below
 * 2^-22.  x, y: device float [n]; asynchronous on `stream`; SPATTEN_E_ARG for NULL or n < 1.
 * ============================================================================================= */
int32_t spatten_selftest_exp2_poly(const float* x, float* y, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SPATTEN_H */
