// K3: decode attention -- one query row per (sequence, kept head) against the index-listed cache,
// with progressive quantization and importance.
//
// SpAtten §II "Attention-based NLP models": generation handles one new token per iteration
// against cached K and V (a memory-bound workload); §IV.E "Progressive Quantization": the LSBs
// are fetched only when the max probability is below the threshold.
// Per CTA (b, kept head):
//   1  MSB scores: lanes read 16-byte slices of the int8 MSB rows (d_h/16 lanes per key, rows
//      reached through kv_idx), s_j = (16 * s_k * sm_scale) * (q . MSB_j); kept in shared memory.
//   2  row stats m, ell; flag = 1/ell < theta.
//   3  flagged rows only: read the LSB rows, s_j += s_k * sm_scale * (q . LSB_j); new m, ell.
//   4  p_j = exp(s_j - m)/ell -> importance partial; O = s_v * sum_j p_j (16*MSB_j [+ LSB_j]).
// Every sweep over the keys issues kUnroll independent index loads and then kUnroll independent
// 16-byte row loads per lane before using them, so each CTA keeps tens of KB in flight (the sweep
// is bound by HBM bandwidth, not by load latency).  Importance partials are reduced over heads
// in a fixed order by attn_reduce.
#include "attention.cuh"

namespace spt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxKv = 32768;   // scores kept in shared memory (128 KB)
constexpr int kUnroll = 4;

__device__ __forceinline__ void unpack16_s8(uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) f[4 * i + k] = static_cast<float>(static_cast<int8_t>((w[i] >> (8 * k)) & 0xFFu));
}
__device__ __forceinline__ void unpack16_u4(uint2 u, float* f) {
  const uint32_t w[2] = {u.x, u.y};
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) f[8 * i + k] = static_cast<float>((w[i] >> (4 * k)) & 0xFu);
}

template <int DH, typename QT>
__global__ void __launch_bounds__(kThreads) attn_decode_kernel(AttnProblem p) {
  const spatten_attn_args& a = p.a;
  constexpr int LPK = DH / 16;          // lanes per key row (16 codes per lane)
  constexpr int KPW = 32 / LPK;         // keys per warp per step
  constexpr int KPS = KPW * kWarps;     // keys per CTA step
  constexpr int KPU = KPS * kUnroll;    // keys per unrolled step
  extern __shared__ __align__(16) float s_sc[];   // [n_kv] scores, then probabilities
  __shared__ float red[kWarps];
  __shared__ float o_red[kWarps][DH];
  __shared__ float bcast[2];

  const int slot = blockIdx.x, b = blockIdx.y;
  const int h = head_of_slot(a, b, slot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPK, grp = lane / LPK;
  QT* o = static_cast<QT*>(a.o);
  if (slot >= a.H_kept) {
    if (h >= 0 && threadIdx.x < DH)
      st_from_float(o + static_cast<int64_t>(b) * a.n_q * a.o_ld_tok + static_cast<int64_t>(h) * DH + threadIdx.x, 0.0f);
    return;
  }
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t plane0 = bh * a.kv_cap;
  const int32_t* kv_idx = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;

  float qf[16];
  {
    const QT* q = static_cast<const QT*>(a.q) + static_cast<int64_t>(b) * a.n_q * a.q_ld_tok + static_cast<int64_t>(h) * DH + sub * 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) qf[i] = ld_as_float(q + i);
  }
  const float ks = a.k_scale[bh], vs = a.v_scale[bh];
  const float c_msb = 16.0f * ks * a.sm_scale;
  const float c_lsb = ks * a.sm_scale;
  const int n = a.n_kv;

  // rows of the kUnroll keys this lane group handles in the unrolled step starting at j0
  auto rows_of = [&](int j0, int64_t* rows, int* js) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      js[u] = j0 + u * KPS + warp * KPW + grp;
      rows[u] = js[u] < n ? plane0 + (kv_idx ? __ldg(kv_idx + js[u]) : js[u]) : 0;
    }
  };

  // ---- 1: MSB scores -------------------------------------------------------------------------
  float mloc = -INFINITY;
  for (int j0 = 0; j0 < n; j0 += KPU) {
    int64_t rows[kUnroll];
    int js[kUnroll];
    rows_of(j0, rows, js);
    uint4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      raw[u] = js[u] < n ? __ldg(reinterpret_cast<const uint4*>(a.k_msb + rows[u] * DH) + sub) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float f[16];
      unpack16_s8(raw[u], f);
      float part = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) part = fmaf(qf[i], f[i], part);
#pragma unroll
      for (int o2 = 1; o2 < LPK; o2 <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
      if (js[u] < n && sub == 0) {
        const float s = part * c_msb;
        s_sc[js[u]] = s;
        mloc = fmaxf(mloc, s);
      }
    }
  }
  auto block_max = [&](float v) {
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = red[0];
      for (int w = 1; w < kWarps; ++w) t = fmaxf(t, red[w]);
      bcast[0] = t;
    }
    __syncthreads();
    return bcast[0];
  };
  auto block_sum = [&](float v) {
    v = warp_sum(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.0f;
      for (int w = 0; w < kWarps; ++w) t += red[w];
      bcast[1] = t;
    }
    __syncthreads();
    return bcast[1];
  };
  __syncthreads();
  float m = block_max(mloc);
  float l = 0.0f;
  for (int j = threadIdx.x; j < n; j += kThreads) l += expf(s_sc[j] - m);
  l = block_sum(l);
  const bool flag = 1.0f / l < a.refetch_threshold;

  // ---- 3: LSB refetch for a flagged row ------------------------------------------------------
  if (flag) {
    mloc = -INFINITY;
    for (int j0 = 0; j0 < n; j0 += KPU) {
      int64_t rows[kUnroll];
      int js[kUnroll];
      rows_of(j0, rows, js);
      uint2 raw[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        raw[u] = js[u] < n ? __ldg(reinterpret_cast<const uint2*>(a.k_lsb + rows[u] * (DH / 2)) + sub) : make_uint2(0, 0);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        float f[16];
        unpack16_u4(raw[u], f);
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) part = fmaf(qf[i], f[i], part);
#pragma unroll
        for (int o2 = 1; o2 < LPK; o2 <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
        if (js[u] < n && sub == 0) {
          const float s = s_sc[js[u]] + part * c_lsb;
          s_sc[js[u]] = s;
          mloc = fmaxf(mloc, s);
        }
      }
    }
    __syncthreads();
    m = block_max(mloc);
    l = 0.0f;
    for (int j = threadIdx.x; j < n; j += kThreads) l += expf(s_sc[j] - m);
    l = block_sum(l);
  }
  const float inv_l = 1.0f / l;

  // ---- 4: probabilities, importance partial, output ------------------------------------------
  float* part_row = p.tok_part + (static_cast<int64_t>(b) * a.H_kept + slot) * a.n_kv;
  for (int j = threadIdx.x; j < n; j += kThreads) {
    const float pr = expf(s_sc[j] - m) * inv_l;
    s_sc[j] = pr;
    part_row[j] = pr;
  }
  __syncthreads();
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
  for (int j0 = 0; j0 < n; j0 += KPU) {
    int64_t rows[kUnroll];
    int js[kUnroll];
    rows_of(j0, rows, js);
    uint4 rm[kUnroll];
    uint2 rl[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      rm[u] = js[u] < n ? __ldg(reinterpret_cast<const uint4*>(a.v_msb + rows[u] * DH) + sub) : make_uint4(0, 0, 0, 0);
      rl[u] = (flag && js[u] < n) ? __ldg(reinterpret_cast<const uint2*>(a.v_lsb + rows[u] * (DH / 2)) + sub) : make_uint2(0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (js[u] >= n) continue;
      const float pr = s_sc[js[u]];
      float f[16], g[16];
      unpack16_s8(rm[u], f);
      unpack16_u4(rl[u], g);   // zero unless the row refetches
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = fmaf(pr, fmaf(16.0f, f[i], g[i]), acc[i]);
    }
  }
  // reduce over the key groups of the warp (lanes with equal `sub`), then over warps
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int o2 = LPK; o2 < 32; o2 <<= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o2);
  if (grp == 0) {
#pragma unroll
    for (int i = 0; i < 16; ++i) o_red[warp][sub * 16 + i] = acc[i];
  }
  __syncthreads();
  float habs = 0.0f;
  if (threadIdx.x < DH) {
    float v = 0.0f;
    for (int w = 0; w < kWarps; ++w) v += o_red[w][threadIdx.x];
    v *= vs;
    habs = fabsf(v);
    st_from_float(o + static_cast<int64_t>(b) * a.n_q * a.o_ld_tok + static_cast<int64_t>(h) * DH + threadIdx.x, v);
  }
  habs = block_sum(habs);
  if (threadIdx.x == 0) {
    p.head_part[static_cast<int64_t>(b) * a.H_kept + slot] = habs;
    if (a.refetch_flags) a.refetch_flags[bh * a.refetch_flags_ld] = flag ? 1 : 0;
    if (flag && a.refetch_count) atomicAdd(a.refetch_count, 1);
  }
}

template <int DH, typename QT>
int32_t launch(const AttnProblem& p, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    SPT_CUDA(cudaFuncSetAttribute(attn_decode_kernel<DH, QT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxKv * 4));
    configured[dev] = true;
  }
  const int slots = p.a.H_kept + (p.a.zero_pruned_heads ? p.a.H - p.a.H_kept : 0);
  const size_t smem = static_cast<size_t>(p.a.n_kv) * 4;
  attn_decode_kernel<DH, QT><<<dim3(slots, p.a.B), kThreads, smem, st>>>(p);
  return launch_status();
}

}  // namespace

bool attn_decode_supported(const spatten_attn_args& a) {
  return a.quantized && a.n_q == 1 && a.n_kv <= kMaxKv && (a.d_h == 64 || a.d_h == 128);
}

int32_t attn_decode_launch(const AttnProblem& p, cudaStream_t st) {
  const bool bf = p.a.q_dtype == SPATTEN_BF16;
  if (p.a.d_h == 64) return bf ? launch<64, __nv_bfloat16>(p, st) : launch<64, float>(p, st);
  return bf ? launch<128, __nv_bfloat16>(p, st) : launch<128, float>(p, st);
}

}  // namespace spt
