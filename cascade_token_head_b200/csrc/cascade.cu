// spatten_cascade_forward: the per-layer loop of cascade token/head pruning (prefill) and of one
// generation step (decode).
//
// SpAtten §II "Cascade pruning": tokens and heads pruned in one layer stay pruned in every later
// layer; token importance is the cumulative attention probability a token received, head
// importance the cumulative |attention output|; the top-k survive.  §II.B "Motivation": the
// fully-connected layers run off the attention engine -- here on the library GEMM (cuBLASLt),
// everything else in this library's kernels.  The host never reads device memory inside the loop
// (all sizes come from the schedule), so a whole forward can be captured in a CUDA graph.
// The next layer's selections (top-k of the importance vectors) depend on the attention step but
// not on the output projection, so they run on a second stream of the library's own, forked from
// and joined back to the caller's stream by events, overlapping the projection GEMMs.
#include <cublasLt.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "attention.cuh"
#include "common.cuh"

namespace spt {
namespace {

constexpr size_t kGemmWs = 32u << 20;   // cuBLASLt workspace carved from the caller's ws

// ------------------------------------------------------------------------------------------------
// cuBLASLt: C[M,N] (+)= A[M,K] @ W[K,N], all row-major
// ------------------------------------------------------------------------------------------------
struct GemmPlan {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulAlgo_t algo;
  bool ok = false;
};

std::mutex g_gemm_mu;
cublasLtHandle_t g_lt[64] = {nullptr};
std::map<std::tuple<int, int, int, int, int, int>, GemmPlan> g_plans;

int32_t gemm_rm(const void* A, const void* W, void* C, int M, int N, int K, int dtype, bool accumulate,
                void* ws, cudaStream_t st) {
  int dev = 0;
  SPT_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lock(g_gemm_mu);
  if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
  auto key = std::make_tuple(dev, M, N, K, dtype, accumulate ? 1 : 0);
  GemmPlan& p = g_plans[key];
  const cudaDataType_t t = dtype == SPATTEN_BF16 ? CUDA_R_16BF : CUDA_R_32F;
  if (!p.ok) {
    // column-major view: D^T[N,M] = W^T[N,K] @ A^T[K,M]
    const cublasComputeType_t ct = CUBLAS_COMPUTE_32F;   // full float32 accumulation (no TF32)
    if (cublasLtMatmulDescCreate(&p.op, ct, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
    if (cublasLtMatrixLayoutCreate(&p.la, t, N, K, N) != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
    if (cublasLtMatrixLayoutCreate(&p.lb, t, K, M, K) != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
    if (cublasLtMatrixLayoutCreate(&p.lc, t, N, M, N) != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
    cublasLtMatmulPreference_t pref;
    if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
    size_t wsz = kGemmWs;
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &wsz, sizeof(wsz));
    cublasLtMatmulHeuristicResult_t res;
    int found = 0;
    cublasStatus_t hs = cublasLtMatmulAlgoGetHeuristic(g_lt[dev], p.op, p.la, p.lb, p.lc, p.lc, pref, 1, &res, &found);
    cublasLtMatmulPreferenceDestroy(pref);
    if (hs != CUBLAS_STATUS_SUCCESS || found < 1) return SPATTEN_E_UNSUPPORTED;
    p.algo = res.algo;
    p.ok = true;
  }
  const float alpha = 1.0f, beta = accumulate ? 1.0f : 0.0f;
  cublasStatus_t s = cublasLtMatmul(g_lt[dev], p.op, &alpha, W, p.la, A, p.lb, &beta, C, p.lc, C, p.lc,
                                    &p.algo, ws, kGemmWs, st);
  if (s != CUBLAS_STATUS_SUCCESS) return SPATTEN_E_CUDA;
  return SPATTEN_OK;
}

// ------------------------------------------------------------------------------------------------
// small helper kernels
// ------------------------------------------------------------------------------------------------
__global__ void iota_rows_kernel(int32_t* out, int64_t ld, int n) {
  const int r = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < n; j += gridDim.x * blockDim.x)
    out[static_cast<int64_t>(r) * ld + j] = j;
}

int32_t iota_rows(int32_t* out, int64_t ld, int n, int R, cudaStream_t st) {
  iota_rows_kernel<<<dim3(static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 64)), R), 256, 0, st>>>(out, ld, n);
  return launch_status();
}

int32_t copy2d(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, size_t rows,
               cudaStream_t st) {
  if (width == 0 || rows == 0) return SPATTEN_OK;
  SPT_CUDA(cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, cudaMemcpyDeviceToDevice, st));
  return SPATTEN_OK;
}

int esize(int dtype) { return dtype == SPATTEN_BF16 ? 2 : 4; }

cudaEvent_t ev(const spatten_cascade_io& io, int i) {
  return io.attn_events ? static_cast<cudaEvent_t>(io.attn_events[i]) : nullptr;
}

// workspace layout (identical for the size query and the run)
struct Ws {
  char* xa; char* xb; char* qkv; char* o;
  int8_t* k_msb; int8_t* v_msb; uint8_t* k_lsb; uint8_t* v_lsb; float* k_scale; float* v_scale;
  float* gain_a; float* gain_b;
  int32_t* sel; int32_t* head_sel;
  void* attn_ws; size_t attn_ws_bytes;
  void* gemm_ws;
  size_t total;
};

// the largest workspace any attention kernel asks for at this size (sizes grow with n and the
// number of kept heads, so layer 0 bounds every layer)
size_t attn_ws_bound(const spatten_cascade_cfg& c, int n_q, int n_kv) {
  spatten_attn_args a;
  std::memset(&a, 0, sizeof(a));
  void* const dummy = reinterpret_cast<void*>(uintptr_t(256));   // sizing only, never dereferenced
  a.B = c.B; a.H = c.H; a.n_q = n_q; a.n_kv = n_kv; a.d_h = c.d_h; a.H_kept = c.H;
  a.q = dummy; a.o = dummy; a.q_dtype = c.dtype;
  a.q_ld_tok = 3LL * c.H * c.d_h; a.o_ld_tok = static_cast<int64_t>(c.H) * c.d_h;
  a.quantized = c.quant;
  a.k_msb = a.v_msb = static_cast<const int8_t*>(dummy);
  a.k_lsb = a.v_lsb = static_cast<const uint8_t*>(dummy);
  a.k_scale = a.v_scale = static_cast<const float*>(dummy);
  a.kv_cap = n_kv;
  a.k = a.v = dummy; a.kv_dtype = c.dtype; a.kv_ld_tok = a.q_ld_tok;
  size_t best = 0;
  for (int kernel = SPATTEN_ATTN_AUTO; kernel <= SPATTEN_ATTN_DECODE; ++kernel) {
    a.kernel = kernel;
    best = std::max(best, spatten_attention_workspace_size(&a));
  }
  return best + 512;
}

Ws carve(const spatten_cascade_cfg& c, void* base) {
  Ws w{};
  WsCursor cur(base, ~size_t(0));
  const size_t es = esize(c.dtype);
  const bool dec = c.mode == SPATTEN_DECODE_STEP;
  const size_t rows = dec ? static_cast<size_t>(c.B) : static_cast<size_t>(c.B) * c.T;
  const size_t HD = static_cast<size_t>(c.H) * c.d_h;
  w.xa = cur.take<char>(rows * c.D * es);
  w.xb = cur.take<char>(rows * c.D * es);
  w.qkv = cur.take<char>(rows * 3 * HD * es);
  w.o = cur.take<char>(rows * HD * es);
  if (!dec && c.quant) {
    const size_t planes = static_cast<size_t>(c.B) * c.H * c.T * c.d_h;
    w.k_msb = cur.take<int8_t>(planes);
    w.v_msb = cur.take<int8_t>(planes);
    w.k_lsb = cur.take<uint8_t>(planes / 2);
    w.v_lsb = cur.take<uint8_t>(planes / 2);
    w.k_scale = cur.take<float>(static_cast<size_t>(c.B) * c.H);
    w.v_scale = cur.take<float>(static_cast<size_t>(c.B) * c.H);
  }
  if (!dec) {
    w.gain_a = cur.take<float>(static_cast<size_t>(c.B) * c.T);
    w.gain_b = cur.take<float>(static_cast<size_t>(c.B) * c.T);
  }
  w.sel = cur.take<int32_t>(static_cast<size_t>(c.B) * c.T);
  w.head_sel = cur.take<int32_t>(static_cast<size_t>(c.B) * c.H);
  w.attn_ws_bytes = dec ? attn_ws_bound(c, 1, c.T) : attn_ws_bound(c, c.T, c.T);
  w.attn_ws = cur.take<char>(w.attn_ws_bytes);
  w.gemm_ws = cur.take<char>(kGemmWs);
  w.total = cur.used;
  return w;
}

int32_t validate_cfg(const spatten_cascade_cfg& c) {
  if (c.mode != SPATTEN_PREFILL && c.mode != SPATTEN_DECODE_STEP) return SPATTEN_E_ARG;
  if (c.B < 1 || c.T < 1 || c.D < 1 || c.H < 1 || c.L < 1 || c.L > SPATTEN_MAX_LAYERS) return SPATTEN_E_ARG;
  if (c.B > 65535) return SPATTEN_E_ARG;
  if (c.d_h != 64 && c.d_h != 128) return SPATTEN_E_UNSUPPORTED;
  if (c.dtype != SPATTEN_F32 && c.dtype != SPATTEN_BF16) return SPATTEN_E_ARG;
  if (c.D % 8 != 0) return SPATTEN_E_ALIGN;
  if (c.token_keep[0] != c.T) return SPATTEN_E_SHAPE;
  for (int l = 0; l < c.L; ++l) {
    if (c.token_keep[l] < 1 || (l > 0 && c.token_keep[l] > c.token_keep[l - 1])) return SPATTEN_E_SHAPE;
    const int hk = c.mode == SPATTEN_DECODE_STEP ? c.H : c.head_keep[l];
    if (hk < 1 || hk > c.H || (l > 0 && c.mode == SPATTEN_PREFILL && hk > c.head_keep[l - 1])) return SPATTEN_E_SHAPE;
  }
  if (c.mode == SPATTEN_PREFILL && c.head_keep[0] != c.H) return SPATTEN_E_SHAPE;
  if (c.mode == SPATTEN_DECODE_STEP && !c.quant) return SPATTEN_E_UNSUPPORTED;
  return SPATTEN_OK;
}

spatten_attn_args base_attn(const spatten_cascade_cfg& c) {
  spatten_attn_args a;
  std::memset(&a, 0, sizeof(a));
  a.B = c.B;
  a.H = c.H;
  a.d_h = c.d_h;
  a.q_dtype = c.dtype;
  a.sm_scale = c.sm_scale;
  a.refetch_threshold = c.refetch_threshold;
  a.zero_pruned_heads = 1;
  return a;
}

// ------------------------------------------------------------------------------------------------
// side stream: one per device and host thread, created on the first call outside a stream capture
// (creating a stream inside one is not allowed; such a call runs its selections on the caller's
// stream instead)
// ------------------------------------------------------------------------------------------------
struct Side {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaStream_t origin = nullptr;   // the stream forked from; null when running on it
  cudaStream_t use(cudaStream_t st) const { return origin ? s : st; }
};

int32_t side_fork(cudaStream_t st, Side** out) {
  thread_local Side sides[64];
  *out = nullptr;
  int dev = 0;
  SPT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return SPATTEN_OK;
  Side& sd = sides[dev];
  sd.origin = nullptr;
  *out = &sd;
  if (!sd.s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    SPT_CUDA(cudaStreamIsCapturing(st, &cs));
    if (cs != cudaStreamCaptureStatusNone) return SPATTEN_OK;
    SPT_CUDA(cudaStreamCreateWithFlags(&sd.s, cudaStreamNonBlocking));
    SPT_CUDA(cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming));
    SPT_CUDA(cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming));
  }
  SPT_CUDA(cudaEventRecord(sd.fork, st));
  SPT_CUDA(cudaStreamWaitEvent(sd.s, sd.fork, 0));
  sd.origin = st;
  return SPATTEN_OK;
}

int32_t side_join(Side* sd) {
  if (!sd || !sd->origin) return SPATTEN_OK;
  SPT_CUDA(cudaEventRecord(sd->join, sd->s));
  SPT_CUDA(cudaStreamWaitEvent(sd->origin, sd->join, 0));
  sd->origin = nullptr;
  return SPATTEN_OK;
}

// joins an open fork when the forward leaves early (an error), so that no stream capture is left
// with an unjoined stream
struct SideGuard {
  Side*& sd;
  ~SideGuard() {
    if (sd) side_join(sd);
  }
};

// ------------------------------------------------------------------------------------------------
// prefill
// ------------------------------------------------------------------------------------------------
int32_t run_prefill(const spatten_cascade_cfg& c, const spatten_layer_weights* w, spatten_cascade_io& io,
                    const Ws& ws, cudaStream_t st) {
  const int B = c.B, T = c.T, D = c.D, H = c.H, dh = c.d_h, L = c.L;
  const int64_t HD = static_cast<int64_t>(H) * dh;
  const size_t es = esize(c.dtype);
  SPT_CUDA(cudaMemsetAsync(io.tok_imp, 0, sizeof(float) * B * T, st));
  SPT_CUDA(cudaMemsetAsync(io.head_imp, 0, sizeof(float) * B * H, st));
  SPT_CUDA(cudaMemsetAsync(io.refetch_count, 0, sizeof(int32_t) * L, st));
  SPT_TRY(iota_rows(io.kept_tok, T, T, B, st));
  SPT_TRY(iota_rows(io.kept_head, H, H, B, st));
  SPT_CUDA(cudaMemcpyAsync(ws.xa, io.x, static_cast<size_t>(B) * T * D * es, cudaMemcpyDeviceToDevice, st));
  const bool gain = io.key_gain != nullptr;
  if (gain) SPT_CUDA(cudaMemcpyAsync(ws.gain_a, io.key_gain, sizeof(float) * B * T, cudaMemcpyDeviceToDevice, st));

  char* cur = ws.xa;
  char* nxt = ws.xb;
  float* g_cur = ws.gain_a;
  float* g_nxt = ws.gain_b;
  Side* side = nullptr;
  SideGuard guard{side};
  for (int l = 0; l < L; ++l) {
    const int k = c.token_keep[l], Hl = c.head_keep[l];
    int32_t* kept_l = io.kept_tok + static_cast<int64_t>(l) * B * T;
    int32_t* khead_l = io.kept_head + static_cast<int64_t>(l) * B * H;
    if (io.trace_x)
      SPT_TRY(copy2d(static_cast<char*>(io.trace_x) + static_cast<size_t>(l) * B * T * D * es, T * D * es, cur,
                     k * D * es, k * D * es, B, st));
    // projections of the kept rows (all heads): qkv[B*k, 3HD] = X[B*k, D] @ W_qkv
    SPT_TRY(gemm_rm(cur, w[l].w_qkv, ws.qkv, B * k, static_cast<int>(3 * HD), D, c.dtype, false, ws.gemm_ws, st));
    if (io.trace_qkv)
      SPT_TRY(copy2d(static_cast<char*>(io.trace_qkv) + static_cast<size_t>(l) * B * T * 3 * HD * es, T * 3 * HD * es,
                     ws.qkv, k * 3 * HD * es, k * 3 * HD * es, B, st));
    spatten_attn_args a = base_attn(c);
    a.n_q = k;
    a.n_kv = k;
    a.H_kept = Hl;
    a.head_idx = khead_l;
    a.head_idx_ld = H;
    a.q = ws.qkv;
    a.q_ld_tok = 3 * HD;
    if (c.quant) {
      const char* kp = ws.qkv + HD * es;
      const char* vp = ws.qkv + 2 * HD * es;
      SPT_TRY(quantize_kv_pair(kp, vp, c.dtype, B, H, k, dh, 3 * HD, gain ? g_cur : nullptr, k, nullptr, nullptr,
                               ws.k_msb, ws.k_lsb, ws.v_msb, ws.v_lsb, k, 0, ws.k_scale, ws.v_scale, nullptr, st));
      a.quantized = 1;
      a.k_msb = ws.k_msb; a.k_lsb = ws.k_lsb; a.k_scale = ws.k_scale;
      a.v_msb = ws.v_msb; a.v_lsb = ws.v_lsb; a.v_scale = ws.v_scale;
      a.kv_cap = k;
    } else {
      if (gain) return SPATTEN_E_UNSUPPORTED;
      a.quantized = 0;
      a.k = ws.qkv + HD * es;
      a.v = ws.qkv + 2 * HD * es;
      a.kv_dtype = c.dtype;
      a.kv_ld_tok = 3 * HD;
    }
    a.o = ws.o;
    a.o_ld_tok = HD;
    a.tok_imp = io.tok_imp;
    a.tok_imp_ld = T;
    a.tok_imp_map = kept_l;
    a.tok_imp_map_ld = T;
    a.head_imp = io.head_imp;
    a.refetch_flags = io.trace_flags ? io.trace_flags + static_cast<int64_t>(l) * B * H * T : nullptr;
    a.refetch_flags_ld = T;
    a.refetch_count = io.refetch_count + l;
    a.dev_status = io.dev_status;
    SPT_TRY(attention_layer_timed(&a, ws.attn_ws, ws.attn_ws_bytes, st, ev(io, 2 * l), ev(io, 2 * l + 1)));
    if (io.trace_o)
      SPT_TRY(copy2d(static_cast<char*>(io.trace_o) + static_cast<size_t>(l) * B * T * HD * es, T * HD * es, ws.o,
                     k * HD * es, k * HD * es, B, st));
    if (io.trace_tok_imp)
      SPT_CUDA(cudaMemcpyAsync(io.trace_tok_imp + static_cast<size_t>(l) * B * T, io.tok_imp, sizeof(float) * B * T,
                               cudaMemcpyDeviceToDevice, st));
    if (io.trace_head_imp)
      SPT_CUDA(cudaMemcpyAsync(io.trace_head_imp + static_cast<size_t>(l) * B * H, io.head_imp, sizeof(float) * B * H,
                               cudaMemcpyDeviceToDevice, st));
    const int k2 = l + 1 < L ? c.token_keep[l + 1] : 0;
    if (l + 1 < L) {
      // the next layer's selections, beside the projection: token top-k_{l+1} of the cumulative
      // importance over S_l (read through kept_l), the kept rows' gains, the head selection
      SPT_TRY(side_fork(st, &side));
      const cudaStream_t ss = side ? side->use(st) : st;
      auto select = [&]() -> int32_t {
        int32_t* kept_n = io.kept_tok + static_cast<int64_t>(l + 1) * B * T;
        SPT_TRY(spatten_topk_select(io.tok_imp, B, k, T, k2, kept_l, T, ws.sel, T, kept_n, nullptr, 0, io.dev_status,
                                    ss));
        if (gain)
          SPT_TRY(spatten_gather_kept(g_cur, static_cast<int64_t>(k) * 4, 4, k, 4, B, ws.sel, T, k2, g_nxt,
                                      static_cast<int64_t>(k2) * 4, 4, nullptr, 0, nullptr, 0, nullptr, ss));
        const int H2 = c.head_keep[l + 1];
        int32_t* khead_n = io.kept_head + static_cast<int64_t>(l + 1) * B * H;
        if (H2 < Hl)
          return spatten_topk_select(io.head_imp, B, Hl, H, H2, khead_l, H, ws.head_sel, H, khead_n, nullptr, 0,
                                     io.dev_status, ss);
        SPT_CUDA(cudaMemcpyAsync(khead_n, khead_l, sizeof(int32_t) * B * H, cudaMemcpyDeviceToDevice, ss));
        return SPATTEN_OK;
      };
      SPT_TRY(select());
    }
    // residual: X[B*k, D] += O[B*k, HD] @ W_o   (pruned heads' O are zero)
    SPT_TRY(gemm_rm(ws.o, w[l].w_o, cur, B * k, D, static_cast<int>(HD), c.dtype, true, ws.gemm_ws, st));
    if (l == L - 1) break;
    SPT_TRY(side_join(side));
    side = nullptr;
    SPT_TRY(spatten_gather_kept(cur, static_cast<int64_t>(k) * D * es, D * es, k, D * es, B, ws.sel, T, k2, nxt,
                                static_cast<int64_t>(k2) * D * es, D * es, nullptr, 0, nullptr, 0, nullptr, st));
    std::swap(cur, nxt);
    std::swap(g_cur, g_nxt);
  }
  const int kl = c.token_keep[L - 1];
  SPT_CUDA(cudaMemcpyAsync(io.x_out, cur, static_cast<size_t>(B) * kl * D * es, cudaMemcpyDeviceToDevice, st));
  return SPATTEN_OK;
}

// ------------------------------------------------------------------------------------------------
// decode step
// ------------------------------------------------------------------------------------------------
int32_t run_decode(const spatten_cascade_cfg& c, const spatten_layer_weights* w, spatten_cascade_io& io,
                   const Ws& ws, cudaStream_t st) {
  const int B = c.B, n = c.T, D = c.D, H = c.H, dh = c.d_h, L = c.L, cap = io.cap;
  const int64_t HD = static_cast<int64_t>(H) * dh;
  const size_t es = esize(c.dtype);
  if (io.refetch_count) SPT_CUDA(cudaMemsetAsync(io.refetch_count, 0, sizeof(int32_t) * L, st));
  SPT_TRY(iota_rows(io.kept_tok, cap, n, B, st));
  SPT_CUDA(cudaMemcpyAsync(ws.xa, io.x, static_cast<size_t>(B) * D * es, cudaMemcpyDeviceToDevice, st));
  char* x = ws.xa;
  Side* side = nullptr;   // the previous layer's cache-row selection, beside this layer's projections
  SideGuard guard{side};
  for (int l = 0; l < L; ++l) {
    const int k = c.token_keep[l];
    const spatten_decode_cache& cc = io.caches[l];
    int32_t* kept_l = io.kept_tok + static_cast<int64_t>(l) * B * cap;
    if (io.trace_x)
      SPT_CUDA(cudaMemcpyAsync(static_cast<char*>(io.trace_x) + static_cast<size_t>(l) * B * D * es, x,
                               static_cast<size_t>(B) * D * es, cudaMemcpyDeviceToDevice, st));
    SPT_TRY(gemm_rm(x, w[l].w_qkv, ws.qkv, B, static_cast<int>(3 * HD), D, c.dtype, false, ws.gemm_ws, st));
    if (io.trace_qkv)
      SPT_CUDA(cudaMemcpyAsync(static_cast<char*>(io.trace_qkv) + static_cast<size_t>(l) * B * 3 * HD * es, ws.qkv,
                               static_cast<size_t>(B) * 3 * HD * es, cudaMemcpyDeviceToDevice, st));
    // append the new token's K and V codes at row n-1 with the prompt-time scales
    SPT_TRY(quantize_kv_pair(ws.qkv + HD * es, ws.qkv + 2 * HD * es, c.dtype, B, H, 1, dh, 3 * HD, nullptr, 0,
                             cc.k_scale, cc.v_scale, cc.k_msb, cc.k_lsb, cc.v_msb, cc.v_lsb, cap, io.n_old, nullptr,
                             nullptr, io.sat_count, st));
    spatten_attn_args a = base_attn(c);
    a.n_q = 1;
    a.n_kv = k;
    a.H_kept = H;
    a.q = ws.qkv;
    a.q_ld_tok = 3 * HD;
    a.quantized = 1;
    a.k_msb = cc.k_msb; a.k_lsb = cc.k_lsb; a.k_scale = cc.k_scale;
    a.v_msb = cc.v_msb; a.v_lsb = cc.v_lsb; a.v_scale = cc.v_scale;
    a.kv_cap = cap;
    a.kv_idx = kept_l;
    a.kv_idx_ld = cap;
    a.o = ws.o;
    a.o_ld_tok = HD;
    a.tok_imp = io.dec_tok_imp;
    a.tok_imp_ld = cap;
    a.tok_imp_map = kept_l;
    a.tok_imp_map_ld = cap;
    a.head_imp = io.head_imp;
    a.refetch_flags = io.trace_flags ? io.trace_flags + static_cast<int64_t>(l) * B * H : nullptr;
    a.refetch_flags_ld = 1;
    a.refetch_count = io.refetch_count ? io.refetch_count + l : nullptr;
    a.dev_status = io.dev_status;
    SPT_TRY(side_join(side));   // this layer's kept cache rows
    side = nullptr;
    SPT_TRY(attention_layer_timed(&a, ws.attn_ws, ws.attn_ws_bytes, st, ev(io, 2 * l), ev(io, 2 * l + 1)));
    if (io.trace_o)
      SPT_CUDA(cudaMemcpyAsync(static_cast<char*>(io.trace_o) + static_cast<size_t>(l) * B * HD * es, ws.o,
                               static_cast<size_t>(B) * HD * es, cudaMemcpyDeviceToDevice, st));
    if (io.trace_tok_imp)
      SPT_CUDA(cudaMemcpyAsync(io.trace_tok_imp + static_cast<size_t>(l) * B * cap, io.dec_tok_imp,
                               sizeof(float) * B * cap, cudaMemcpyDeviceToDevice, st));
    if (l + 1 < L) {
      // the next layer's kept cache rows, beside this layer's output projection and the next
      // layer's input projection and cache append (joined before the next attention step)
      SPT_TRY(side_fork(st, &side));
      int32_t* kept_n = io.kept_tok + static_cast<int64_t>(l + 1) * B * cap;
      SPT_TRY(spatten_topk_select(io.dec_tok_imp, B, k, cap, c.token_keep[l + 1], kept_l, cap, nullptr, cap, kept_n,
                                  nullptr, 0, io.dev_status, side ? side->use(st) : st));
    }
    SPT_TRY(gemm_rm(ws.o, w[l].w_o, x, B, D, static_cast<int>(HD), c.dtype, true, ws.gemm_ws, st));
  }
  SPT_CUDA(cudaMemcpyAsync(io.x_out, x, static_cast<size_t>(B) * D * es, cudaMemcpyDeviceToDevice, st));
  return SPATTEN_OK;
}

}  // namespace
}  // namespace spt

extern "C" size_t spatten_cascade_workspace_size(const spatten_cascade_cfg* cfg) {
  using namespace spt;
  if (!cfg || validate_cfg(*cfg) != SPATTEN_OK) return 0;
  return carve(*cfg, nullptr).total;
}

extern "C" int32_t spatten_cascade_forward(const spatten_cascade_cfg* cfg, const spatten_layer_weights* w,
                                           spatten_cascade_io* io, void* ws, size_t ws_bytes, void* stream) {
  spt::AbiRange nvtx_range("spatten_cascade_forward");
  using namespace spt;
  if (!cfg || !w || !io) return SPATTEN_E_ARG;
  SPT_TRY(validate_cfg(*cfg));
  for (int l = 0; l < cfg->L; ++l)
    if (!w[l].w_qkv || !w[l].w_o) return SPATTEN_E_ARG;
  if (!io->x || !io->x_out || !io->kept_tok) return SPATTEN_E_ARG;
  const Ws lay = carve(*cfg, ws);
  if (!ws || ws_bytes < lay.total) return SPATTEN_E_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  if (cfg->mode == SPATTEN_PREFILL) {
    if (!io->kept_head || !io->tok_imp || !io->head_imp || !io->refetch_count) return SPATTEN_E_ARG;
    return run_prefill(*cfg, w, *io, lay, st);
  }
  if (!io->caches || !io->dec_tok_imp || io->cap < cfg->T || io->n_old != cfg->T - 1 || io->n_old < 0)
    return SPATTEN_E_ARG;
  for (int l = 0; l < cfg->L; ++l) {
    const spatten_decode_cache& cc = io->caches[l];
    if (!cc.k_msb || !cc.k_lsb || !cc.k_scale || !cc.v_msb || !cc.v_lsb || !cc.v_scale) return SPATTEN_E_ARG;
  }
  return run_decode(*cfg, w, *io, lay, st);
}
