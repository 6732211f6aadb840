// K3: decode attention -- one query row per (sequence, kept head) against the index-listed cache,
// with progressive quantization and importance.
//
// SpAtten §II "Attention-based NLP models": generation handles one new token per iteration
// against cached K and V (a memory-bound workload); §IV.E "Progressive Quantization": the LSBs
// are fetched only when the max probability is below the threshold.
//
// The work of one row (b, kept head) is cut into items of decode_item_rows(d_h) consecutive
// entries of its key list, one warp per item, and finished by a per-sequence combine step:
//
// items kernel (memory-bound, no block-level barrier): a warp streams the K and V code rows of
//   its item once -- lane groups of d_h/16 lanes read 16-byte MSB and 8-byte packed LSB slices,
//   batches of rows in flight together -- and evaluates both precisions the refetch rule can pick:
//   s1 = s_k * sm_scale * 16 (q . MSB_j)            (MSB pass)
//   s2 = s_k * sm_scale (q . (16 MSB_j + LSB_j))     (full 12-bit codes)
//   It writes, per variant, the item's max m, sum ell of exp(s - m), the exponentials
//   e_j = exp(s_j - m) and the item's sum of e_j times the V codes (MSB_j for the MSB pass, whose
//   values are 16 MSB_j; 16 MSB_j + LSB_j for full precision).  With theta <= 0 no row can refetch and only the MSB
//   variant is computed (the LSB planes are not read).
// combine kernel (one CTA row per sequence): folds the item statistics of every kept head in item
//   order into the row's (m, ell) for each variant, takes the refetch decision 1/ell_MSB < theta,
//   and with the chosen variant's factors f_item = exp(m_item - m) / ell forms
//   p_j = e_j f_item(j)           -> token importance (summed over heads in slot order)
//   O   = s_v sum_items f_item o_item -> output, sum |O| -> head importance.
// Both kernels run in fixed orders, so results are bit-reproducible.  Reading the LSB planes with
// the MSB planes (rather than after the decision) costs up to half of the MSB bytes again for rows
// that do not refetch, and saves a dependent second pass over the cache for rows that do.
#include "attention.cuh"

namespace spt {
namespace {

constexpr int kDWarps = 4;        // warps (items) per CTA of the items kernel
#ifndef SPT_DECODE_BATCH
#define SPT_DECODE_BATCH 8
#endif
constexpr int kCThreads = 256;    // threads per CTA of the combine kernel

template <int DH>
struct DGeom {
  static constexpr int LPK = DH / 16;        // lanes per key row (16 codes per lane)
  static constexpr int KPW = 32 / LPK;       // keys per warp step
  static constexpr int ITEM = 8192 / DH;     // keys per item: 128 (d_h 64), 64 (d_h 128)
  static constexpr int STEPS = ITEM / KPW;   // warp steps per item
  static constexpr int BATCH = SPT_DECODE_BATCH;   // steps whose row loads are in flight together
};

// Paired fp32 arithmetic: the sm_100 float2 intrinsics (two lanes per instruction).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// Signed code bytes to floats: each byte, biased to unsigned (x ^ 0x80), is placed in the low
// mantissa byte of 2^23; subtracting 2^23 + 128 leaves the signed value exactly.  Sixteen codes
// (one uint4) give eight pairs, element 2i and 2i+1 in pair i.
__device__ __forceinline__ void msb16(uint4 v, float2* f) {
  const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u, v.w ^ 0x80808080u};
  const float2 bias = make_float2(-8388736.0f, -8388736.0f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = fadd2(make_float2(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540)),
                                 __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7541))), bias);
    f[2 * i + 1] = fadd2(make_float2(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7542)),
                                     __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7543))), bias);
  }
}
// Sixteen packed 4-bit codes (element 2k in bits 8k..8k+3 of the pair of words, element 2k+1 in
// bits 8k+4..8k+7) as eight pairs.
__device__ __forceinline__ void lsb16(uint2 v, float2* f) {
  const float2 bias = make_float2(-8388608.0f, -8388608.0f);
  const uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      f[4 * i + k] = fadd2(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7540 + k)),
                                       __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7540 + k))), bias);
  }
}

template <int DH, typename QT, bool LSB>
__global__ void __launch_bounds__(kDWarps * 32) attn_decode_items_kernel(AttnProblem p) {
  using G = DGeom<DH>;
  constexpr int LPK = G::LPK, KPW = G::KPW, ITEM = G::ITEM, STEPS = G::STEPS, BATCH = G::BATCH;
  constexpr int NV = LSB ? 2 : 1;   // variants: MSB pass [, full precision]
  const spatten_attn_args& a = p.a;
  __shared__ float s_sc[kDWarps][NV][ITEM];         // scores, then exponentials
  __shared__ float s_o[kDWarps][KPW][NV * DH];      // per lane group sums of e * V

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the (kept head, item) pairs of sequence b, numbered head-major, one per warp
  const int w_id = blockIdx.x * kDWarps + warp;
  const int slot = w_id / p.dec_items, item = w_id % p.dec_items;
  if (slot >= a.H_kept) return;   // warps are independent: no block-level barrier follows
  const int b = blockIdx.y;
  const int h = head_of_slot(a, b, slot);
  const int sub = lane % LPK, grp = lane / LPK;
  const int n = a.n_kv;
  const int j0 = item * ITEM;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t plane0 = bh * a.kv_cap;
  const int64_t bs = static_cast<int64_t>(b) * a.H_kept + slot;
  const int32_t* kv_idx = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;

  float2 qf[8];
  {
    const QT* q = static_cast<const QT*>(a.q) + static_cast<int64_t>(b) * a.n_q * a.q_ld_tok +
                  static_cast<int64_t>(h) * DH + sub * 16;
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[i] = make_float2(ld_as_float(q + 2 * i), ld_as_float(q + 2 * i + 1));
  }
  const float ks = a.k_scale[bh];
  const float c1 = 16.0f * ks * a.sm_scale, c2 = ks * a.sm_scale;
  auto row_of = [&](int j) -> int64_t { return j < n ? plane0 + (kv_idx ? __ldg(kv_idx + j) : j) : -1; };

  // ---- scores of both variants -----------------------------------------------------------------
  float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll 1
  for (int s0 = 0; s0 < STEPS; s0 += BATCH) {
    int64_t row[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u) row[u] = row_of(j0 + (s0 + u) * KPW + grp);
    uint4 km[BATCH];
    uint2 kl[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u)
      km[u] = row[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(a.k_msb + row[u] * DH) + sub) : make_uint4(0, 0, 0, 0);
    if (LSB) {
#pragma unroll
      for (int u = 0; u < BATCH; ++u)
        kl[u] = row[u] >= 0 ? __ldg(reinterpret_cast<const uint2*>(a.k_lsb + row[u] * (DH / 2)) + sub) : make_uint2(0, 0);
    }
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      // d1 = q . MSB_j; d2 = q . LSB_j; the full-precision dot product is 16 d1 + d2
      float2 f[8];
      msb16(km[u], f);
      float2 a1 = make_float2(0.0f, 0.0f), a2 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 8; ++i) a1 = ffma2(qf[i], f[i], a1);
      if (LSB) {
        float2 g[8];
        lsb16(kl[u], g);
#pragma unroll
        for (int i = 0; i < 8; ++i) a2 = ffma2(qf[i], g[i], a2);
      }
      float d1 = a1.x + a1.y, d2 = a2.x + a2.y;
#pragma unroll
      for (int o2 = 1; o2 < LPK; o2 <<= 1) {
        d1 += __shfl_xor_sync(0xffffffffu, d1, o2);
        if (LSB) d2 += __shfl_xor_sync(0xffffffffu, d2, o2);
      }
      if (row[u] >= 0) {
        const float s1 = d1 * c1, s2 = fmaf(16.0f, d1, d2) * c2;
        m1 = fmaxf(m1, s1);
        if (LSB) m2 = fmaxf(m2, s2);
        if (sub == 0) {
          s_sc[warp][0][(s0 + u) * KPW + grp] = s1;
          if (LSB) s_sc[warp][NV - 1][(s0 + u) * KPW + grp] = s2;
        }
      }
    }
  }
  m1 = warp_max(m1);
  if (LSB) m2 = warp_max(m2);
  __syncwarp();

  // ---- exponentials, once per key and variant (coalesced stores) --------------------------------
  const int64_t vstride = static_cast<int64_t>(a.B) * a.H_kept * n;
  float* e_out = p.dec_e + bs * n;
  float l1 = 0.0f, l2 = 0.0f;
  for (int k = lane; k < ITEM; k += 32) {
    const int j = j0 + k;
    if (j < n) {
      const float e1 = expf(s_sc[warp][0][k] - m1);
      s_sc[warp][0][k] = e1;
      e_out[j] = e1;
      l1 += e1;
      if (LSB) {
        const float e2 = expf(s_sc[warp][NV - 1][k] - m2);
        s_sc[warp][NV - 1][k] = e2;
        e_out[vstride + j] = e2;
        l2 += e2;
      }
    }
  }
  l1 = warp_sum(l1);
  if (LSB) l2 = warp_sum(l2);
  __syncwarp();

  // ---- sums of e * V codes ----------------------------------------------------------------------
  float2 o1[8], o2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o1[i] = o2[i] = make_float2(0.0f, 0.0f);
#pragma unroll 1
  for (int s0 = 0; s0 < STEPS; s0 += BATCH) {
    int64_t row[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u) row[u] = row_of(j0 + (s0 + u) * KPW + grp);
    uint4 vm[BATCH];
    uint2 vl[BATCH];
#pragma unroll
    for (int u = 0; u < BATCH; ++u)
      vm[u] = row[u] >= 0 ? __ldg(reinterpret_cast<const uint4*>(a.v_msb + row[u] * DH) + sub) : make_uint4(0, 0, 0, 0);
    if (LSB) {
#pragma unroll
      for (int u = 0; u < BATCH; ++u)
        vl[u] = row[u] >= 0 ? __ldg(reinterpret_cast<const uint2*>(a.v_lsb + row[u] * (DH / 2)) + sub) : make_uint2(0, 0);
    }
#pragma unroll
    for (int u = 0; u < BATCH; ++u) {
      if (row[u] < 0) continue;
      const int k = (s0 + u) * KPW + grp;
      float2 f[8];
      msb16(vm[u], f);
      const float e1 = s_sc[warp][0][k];
      const float2 e1v = make_float2(e1, e1);
#pragma unroll
      for (int i = 0; i < 8; ++i) o1[i] = ffma2(e1v, f[i], o1[i]);
      if (LSB) {
        float2 g[8];
        lsb16(vl[u], g);
        const float e2 = s_sc[warp][NV - 1][k];
        const float2 e2v = make_float2(e2, e2), sixteen = make_float2(16.0f, 16.0f);
#pragma unroll
        for (int i = 0; i < 8; ++i) o2[i] = ffma2(e2v, ffma2(sixteen, f[i], g[i]), o2[i]);
      }
    }
  }
  // add the lane groups' sums through shared memory, in group order
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_o[warp][grp][sub * 16 + 2 * i] = o1[i].x;
    s_o[warp][grp][sub * 16 + 2 * i + 1] = o1[i].y;
    if (LSB) {
      s_o[warp][grp][DH + sub * 16 + 2 * i] = o2[i].x;
      s_o[warp][grp][DH + sub * 16 + 2 * i + 1] = o2[i].y;
    }
  }
  __syncwarp();
  float* o_out = p.dec_o + (bs * p.dec_items + item) * 2 * DH;
  for (int t = lane; t < NV * DH; t += 32) {
    float v = 0.0f;
#pragma unroll
    for (int g = 0; g < KPW; ++g) v += s_o[warp][g][t];
    o_out[t] = v;
  }
  if (lane == 0)
    reinterpret_cast<float4*>(p.dec_stat)[bs * p.dec_items + item] = make_float4(m1, l1, LSB ? m2 : m1, LSB ? l2 : l1);
}

// Row statistics of one kept head folded by one warp in a fixed order (lane-strided item partials,
// then a butterfly); returns whether the row refetches, and the chosen variant's (m, 1/ell).
template <bool LSB>
__device__ __forceinline__ bool fold_row(const float4* st, int NI, float theta, float* m_out, float* inv_l_out) {
  const int lane = threadIdx.x & 31;
  float M1 = -INFINITY, M2 = -INFINITY;
  for (int i = lane; i < NI; i += 32) {
    const float4 v = st[i];
    M1 = fmaxf(M1, v.x);
    M2 = fmaxf(M2, v.z);
  }
  M1 = warp_max(M1);
  if (LSB) M2 = warp_max(M2);
  float L1 = 0.0f, L2 = 0.0f;
  for (int i = lane; i < NI; i += 32) {
    const float4 v = st[i];
    L1 += v.y * expf(v.x - M1);
    if (LSB) L2 += v.w * expf(v.z - M2);
  }
  L1 = warp_sum(L1);
  if (LSB) L2 = warp_sum(L2);
  const bool full = LSB && (1.0f / L1 < theta);
  *m_out = full ? M2 : M1;
  *inv_l_out = 1.0f / (full ? L2 : L1);
  return full;
}

constexpr int kCWarps = kCThreads / 32;

template <int DH, typename QT, bool LSB>
__global__ void __launch_bounds__(kCThreads) attn_decode_combine_kernel(AttnProblem p) {
  constexpr int ITEM = DGeom<DH>::ITEM;
  constexpr int IG = kCThreads / DH;                     // item groups of an output block
  constexpr int TI = (kCThreads + ITEM - 1) / ITEM + 1;  // items a token block can touch
  const spatten_attn_args& a = p.a;
  extern __shared__ float sh[];
  __shared__ float part[IG][DH];
  __shared__ float red[kCWarps];
  const int HK = a.H_kept, NI = p.dec_items, n = a.n_kv;
  const int b = blockIdx.y;
  const int nblk = (n + kCThreads - 1) / kCThreads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4* stats = reinterpret_cast<const float4*>(p.dec_stat) + static_cast<int64_t>(b) * HK * NI;

  if (static_cast<int>(blockIdx.x) < nblk) {
    // ---- token importance of keys [j0, j0 + kCThreads): p_j summed over kept heads in slot order
    // (and, under local value pruning, each head's p_j on its own into head_col)
    if (!a.tok_imp && !p.head_col) return;
    const int j0 = blockIdx.x * kCThreads;
    const int it0 = j0 / ITEM;
    float* factor = sh;                                   // [HK][TI] factors of items it0 ..
    int* use_full = reinterpret_cast<int*>(sh + HK * TI); // [HK]
    for (int slot = warp; slot < HK; slot += kCWarps) {
      float m, inv_l;
      const bool full = fold_row<LSB>(stats + static_cast<int64_t>(slot) * NI, NI, a.refetch_threshold, &m, &inv_l);
      if (lane < TI && it0 + lane < NI) {
        const float4 v = stats[static_cast<int64_t>(slot) * NI + it0 + lane];
        factor[slot * TI + lane] = expf((full ? v.z : v.x) - m) * inv_l;
      }
      if (lane == 0) use_full[slot] = full ? 1 : 0;
    }
    __syncthreads();
    const int j = j0 + threadIdx.x;
    if (j >= n) return;
    const int it = j / ITEM - it0;
    const int64_t vstride = static_cast<int64_t>(a.B) * HK * n;
    const float* e = p.dec_e + static_cast<int64_t>(b) * HK * n + j;
    float t = 0.0f;
    float* hc = p.head_col ? p.head_col + static_cast<int64_t>(b) * HK * n + j : nullptr;
#pragma unroll 4
    for (int slot = 0; slot < HK; ++slot) {
      const float pj = e[(use_full[slot] ? vstride : 0) + static_cast<int64_t>(slot) * n] * factor[slot * TI + it];
      t += pj;
      if (hc) hc[static_cast<int64_t>(slot) * n] = pj;
    }
    if (a.tok_imp) {
      const int64_t col = a.tok_imp_map ? a.tok_imp_map[static_cast<int64_t>(b) * a.tok_imp_map_ld + j] : j;
      a.tok_imp[static_cast<int64_t>(b) * a.tok_imp_ld + col] += t;
    }
    return;
  }
  if (p.v_sel) return;   // local value pruning: the pruned-output kernel writes the outputs

  // ---- output block of one head slot: O, sum |O| -> head importance, refetch flag
  const int slot = static_cast<int>(blockIdx.x) - nblk;
  const int h = head_of_slot(a, b, slot);
  QT* o = static_cast<QT*>(a.o) + static_cast<int64_t>(b) * a.n_q * a.o_ld_tok + static_cast<int64_t>(h) * DH;
  if (slot >= HK) {   // a pruned head: zero-filled output
    if (h >= 0 && threadIdx.x < DH) st_from_float(o + threadIdx.x, 0.0f);
    return;
  }
  float* factor = sh;   // [NI]
  __shared__ int s_full;
  if (warp == 0) {
    float m, inv_l;
    const bool full = fold_row<LSB>(stats + static_cast<int64_t>(slot) * NI, NI, a.refetch_threshold, &m, &inv_l);
    for (int i = lane; i < NI; i += 32) {
      const float4 v = stats[static_cast<int64_t>(slot) * NI + i];
      factor[i] = expf((full ? v.z : v.x) - m) * inv_l;
    }
    if (lane == 0) s_full = full ? 1 : 0;
  }
  __syncthreads();
  const bool full = s_full != 0;
  const int dim = threadIdx.x % DH, g = threadIdx.x / DH;
  {
    const float* op = p.dec_o + (static_cast<int64_t>(b) * HK + slot) * NI * 2 * DH + (full ? DH : 0) + dim;
    float v = 0.0f;
#pragma unroll 4
    for (int i = g; i < NI; i += IG) v += op[static_cast<int64_t>(i) * 2 * DH] * factor[i];
    part[g][dim] = v;
  }
  __syncthreads();
  float absv = 0.0f;
  if (static_cast<int>(threadIdx.x) < DH) {
    float v = 0.0f;
#pragma unroll
    for (int gg = 0; gg < IG; ++gg) v += part[gg][threadIdx.x];
    // the MSB-pass sums hold e * MSB_j; its dequantized value is s_v * 16 * MSB_j
    v *= a.v_scale[static_cast<int64_t>(b) * a.H + h] * (full ? 1.0f : 16.0f);
    st_from_float(o + threadIdx.x, v);
    absv = fabsf(v);
  }
  absv = warp_sum(absv);
  if (lane == 0) red[warp] = absv;
  __syncthreads();
  if (threadIdx.x == 0) {
    float hs = 0.0f;
    for (int w = 0; w < DH / 32; ++w) hs += red[w];
    const int64_t bhh = static_cast<int64_t>(b) * a.H + h;
    if (a.head_imp) a.head_imp[bhh] += hs;
    if (a.refetch_flags) a.refetch_flags[bhh * a.refetch_flags_ld] = full ? 1 : 0;
    if (full && a.refetch_count) atomicAdd(a.refetch_count, 1);
  }
}

// Local value pruning in decode: one CTA per (kept head slot, sequence) [pruned slots: zero fill].
// O = s_v * sum over the v_keep kept keys (ascending, p.v_sel) of p_j * code_j, with p_j the head's
// final probability (p.head_col) and code_j = 16 MSB_j, or 16 MSB_j + LSB_j when the row refetches
// (the same decision as the combine step); groups of threads take keys g, g + G, ... and their
// partial sums are added in group order (bit-reproducible).  Then sum |O| -> head importance, the
// refetch flag and count.
template <int DH, typename QT, bool LSB>
__global__ void __launch_bounds__(kCThreads) attn_decode_pruned_out_kernel(AttnProblem p) {
  constexpr int G = kCThreads / DH;
  const spatten_attn_args& a = p.a;
  const int HK = a.H_kept, NI = p.dec_items, n = a.n_kv;
  const int slot = blockIdx.x, b = blockIdx.y;
  const int h = head_of_slot(a, b, slot);
  QT* o = static_cast<QT*>(a.o) + static_cast<int64_t>(b) * a.n_q * a.o_ld_tok + static_cast<int64_t>(h) * DH;
  if (slot >= HK) {
    if (h >= 0 && threadIdx.x < DH) st_from_float(o + threadIdx.x, 0.0f);
    return;
  }
  __shared__ float part[G][DH];
  __shared__ float red[kCWarps];
  __shared__ int s_full;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float4* stats = reinterpret_cast<const float4*>(p.dec_stat) + (static_cast<int64_t>(b) * HK + slot) * NI;
  if (warp == 0) {
    float m, inv_l;
    const bool full = fold_row<LSB>(stats, NI, a.refetch_threshold, &m, &inv_l);
    if (lane == 0) s_full = full ? 1 : 0;
  }
  __syncthreads();
  const bool full = s_full != 0;
  const int dim = threadIdx.x % DH, g = threadIdx.x / DH;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t plane = bh * a.kv_cap;
  const int32_t* sel = p.v_sel + (static_cast<int64_t>(b) * HK + slot) * a.v_keep;
  const float* pj = p.head_col + (static_cast<int64_t>(b) * HK + slot) * n;
  const int32_t* kvi = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;
  float v = 0.0f;
  for (int c = g; c < a.v_keep; c += G) {
    const int j = sel[c];
    const int64_t row = plane + (kvi ? kvi[j] : j);
    float code = 16.0f * static_cast<float>(a.v_msb[row * DH + dim]);
    if (full) {
      const uint8_t byte = a.v_lsb[row * (DH / 2) + dim / 2];
      code += static_cast<float>((dim & 1) ? (byte >> 4) : (byte & 15));
    }
    v = fmaf(pj[j], code, v);
  }
  part[g][dim] = v;
  __syncthreads();
  float absv = 0.0f;
  if (static_cast<int>(threadIdx.x) < DH) {
    float t = 0.0f;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) t += part[gg][threadIdx.x];
    t *= a.v_scale[bh];
    st_from_float(o + threadIdx.x, t);
    absv = fabsf(t);
  }
  absv = warp_sum(absv);
  if (lane == 0) red[warp] = absv;
  __syncthreads();
  if (threadIdx.x == 0) {
    float hs = 0.0f;
    for (int w = 0; w < DH / 32; ++w) hs += red[w];
    if (a.head_imp) a.head_imp[bh] += hs;
    if (a.refetch_flags) a.refetch_flags[bh * a.refetch_flags_ld] = full ? 1 : 0;
    if (full && a.refetch_count) atomicAdd(a.refetch_count, 1);
  }
}

// dynamic shared memory of the combine kernel: the larger of a token block's factor table and
// flags and an output block's factor row
size_t combine_smem(int d_h, int H_kept, int items) {
  const int item_rows = d_h == 64 ? DGeom<64>::ITEM : DGeom<128>::ITEM;
  const int ti = (kCThreads + item_rows - 1) / item_rows + 1;
  const size_t tok = static_cast<size_t>(H_kept) * (ti + 1) * 4;
  const size_t out = static_cast<size_t>(items) * 4;
  return tok > out ? tok : out;
}

template <int DH, typename QT, bool LSB>
int32_t launch(const AttnProblem& p, cudaStream_t st) {
  const int items = p.dec_items;
  const int64_t per_seq = static_cast<int64_t>(items) * p.a.H_kept;
  attn_decode_items_kernel<DH, QT, LSB>
      <<<dim3(static_cast<unsigned>(ceil_div(per_seq, kDWarps)), p.a.B), kDWarps * 32, 0, st>>>(p);
  SPT_TRY(launch_status());
  const int nblk = static_cast<int>(ceil_div(p.a.n_kv, kCThreads));
  const int slots = p.a.H_kept + (p.a.zero_pruned_heads ? p.a.H - p.a.H_kept : 0);
  attn_decode_combine_kernel<DH, QT, LSB>
      <<<dim3(nblk + slots, p.a.B), kCThreads, combine_smem(DH, p.a.H_kept, items), st>>>(p);
  return launch_status();
}

template <int DH, typename QT>
int32_t launch_dh(const AttnProblem& p, cudaStream_t st) {
  return p.a.refetch_threshold > 0.0f ? launch<DH, QT, true>(p, st) : launch<DH, QT, false>(p, st);
}

template <int DH, typename QT, bool LSB>
int32_t launch_pruned_out(const AttnProblem& p, cudaStream_t st) {
  const int slots = p.a.H_kept + (p.a.zero_pruned_heads ? p.a.H - p.a.H_kept : 0);
  attn_decode_pruned_out_kernel<DH, QT, LSB><<<dim3(slots, p.a.B), kCThreads, 0, st>>>(p);
  return launch_status();
}
template <int DH, typename QT>
int32_t pruned_out_dh(const AttnProblem& p, cudaStream_t st) {
  return p.a.refetch_threshold > 0.0f ? launch_pruned_out<DH, QT, true>(p, st) : launch_pruned_out<DH, QT, false>(p, st);
}

}  // namespace

int decode_item_rows(int d_h) { return d_h == 64 ? DGeom<64>::ITEM : DGeom<128>::ITEM; }

bool attn_decode_supported(const spatten_attn_args& a) {
  if (!a.quantized || a.n_q != 1 || (a.d_h != 64 && a.d_h != 128)) return false;
  // the combine step keeps item factors in shared memory (48 KB without opting in)
  const int64_t items = ceil_div(a.n_kv, decode_item_rows(a.d_h));
  return items <= 12 * 1024 && combine_smem(a.d_h, a.H_kept, static_cast<int>(items)) <= 48 * 1024;
}

int32_t attn_decode_launch(const AttnProblem& p, cudaStream_t st) {
  const bool bf = p.a.q_dtype == SPATTEN_BF16;
  if (p.a.d_h == 64) return bf ? launch_dh<64, __nv_bfloat16>(p, st) : launch_dh<64, float>(p, st);
  return bf ? launch_dh<128, __nv_bfloat16>(p, st) : launch_dh<128, float>(p, st);
}

int32_t attn_decode_pruned_out_launch(const AttnProblem& p, cudaStream_t st) {
  const bool bf = p.a.q_dtype == SPATTEN_BF16;
  if (p.a.d_h == 64) return bf ? pruned_out_dh<64, __nv_bfloat16>(p, st) : pruned_out_dh<64, float>(p, st);
  return bf ? pruned_out_dh<128, __nv_bfloat16>(p, st) : pruned_out_dh<128, float>(p, st);
}

}  // namespace spt
