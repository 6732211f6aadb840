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
// items kernel (memory-bound, no block-level barrier): a warp loads its item's cache rows, then
//   copies every K and V code slice of the item into shared memory at once (cp.async, lane groups
//   of d_h/16 lanes taking 16-byte MSB and 8-byte packed LSB slices of a row; the K copies form
//   one group, the V copies a second, so the scores start while V is still in flight), and
//   evaluates both precisions the refetch rule can pick:
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

constexpr int kDWarps = 2;        // warps (items) per CTA of the items kernel
constexpr int kCThreads = 256;    // threads per CTA of the combine kernel

template <int DH>
struct DGeom {
  static constexpr int LPK = DH / 16;        // lanes per key row (16 codes per lane)
  static constexpr int KPW = 32 / LPK;       // keys per warp step
  static constexpr int ITEM = 8192 / DH;     // keys per item: 128 (d_h 64), 64 (d_h 128)
  static constexpr int STEPS = ITEM / KPW;   // warp steps per item
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

// cp.async copies into shared memory (LDGSTS: no registers held while in flight)
__device__ __forceinline__ uint32_t dsmem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dsmem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dsmem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared memory of one warp of the items kernel: the item's K and V code slices, lane l's slices
// of warp step s at [s][l] (each lane reads back only the slices it copied itself), then the
// scores / exponentials [NV][ITEM]; the lane groups' e * V sums reuse the K MSB area.
template <int DH, bool LSB>
struct DSmem {
  static constexpr int STEPS = DGeom<DH>::STEPS, ITEM = DGeom<DH>::ITEM, KPW = DGeom<DH>::KPW;
  static constexpr int NV = LSB ? 2 : 1;
  static constexpr int kMsb = 0;
  static constexpr int vMsb = kMsb + STEPS * 32 * 16;
  static constexpr int kLsb = vMsb + STEPS * 32 * 16;
  static constexpr int vLsb = kLsb + (LSB ? STEPS * 32 * 8 : 0);
  static constexpr int sc = vLsb + (LSB ? STEPS * 32 * 8 : 0);
  static constexpr int bytes = sc + NV * ITEM * 4;
  static_assert(KPW * NV * DH * 4 <= STEPS * 32 * 16, "the e*V sums fit the K MSB area");
};

// FLAGGED: the full-precision pass of the predicated form, run only for the rows the MSB pass
// flagged (p.dec_flag); it recomputes the MSB variant with the same arithmetic, so the values it
// rewrites are the ones already there
template <int DH, typename QT, bool LSB, bool FLAGGED = false>
__global__ void __launch_bounds__(kDWarps * 32) attn_decode_items_kernel(AttnProblem p) {
  using G = DGeom<DH>;
  using SM = DSmem<DH, LSB>;
  constexpr int LPK = G::LPK, KPW = G::KPW, ITEM = G::ITEM, STEPS = G::STEPS;
  constexpr int NV = SM::NV;
  const spatten_attn_args& a = p.a;
  extern __shared__ __align__(16) unsigned char d_smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the (kept head, item) pairs of sequence b, numbered head-major, one per warp
  const int w_id = blockIdx.x * kDWarps + warp;
  const int slot = w_id / p.dec_items, item = w_id % p.dec_items;
  if (slot >= a.H_kept) return;   // warps are independent: no block-level barrier follows
  if (FLAGGED && !p.dec_flag[static_cast<int64_t>(blockIdx.y) * a.H_kept + slot]) return;
  unsigned char* wsm = d_smem + warp * SM::bytes;
  float* s_sc = reinterpret_cast<float*>(wsm + SM::sc);
  const int b = blockIdx.y;
  const int h = head_of_slot(a, b, slot);
  const int sub = lane % LPK, grp = lane / LPK;
  const int n = a.n_kv;
  const int j0 = item * ITEM;
  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t plane0 = bh * a.kv_cap;
  const int64_t bs = static_cast<int64_t>(b) * a.H_kept + slot;
  const int32_t* kv_idx = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;

  // ---- the item's cache rows (one round trip), then every code slice of the item in flight at
  // once: the K group, then the V group
  int rid[STEPS];   // cache row of the key of step s and this lane group, -1 past the key list
  uint32_t valid = 0;   // bit s: step s has a key
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int j = j0 + s * KPW + grp;
    rid[s] = j < n ? (kv_idx ? __ldg(kv_idx + j) : j) : -1;
    if (j < n) valid |= 1u << s;
  }
  float2 qf[8];
  {
    const QT* q = static_cast<const QT*>(a.q) + static_cast<int64_t>(b) * a.n_q * a.q_ld_tok +
                  static_cast<int64_t>(h) * DH + sub * 16;
#pragma unroll
    for (int i = 0; i < 8; ++i) qf[i] = make_float2(ld_as_float(q + 2 * i), ld_as_float(q + 2 * i + 1));
  }
  const float ks = a.k_scale[bh];
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    if (rid[s] < 0) continue;
    const int64_t r = plane0 + rid[s];
    cp_async16(wsm + SM::kMsb + (s * 32 + lane) * 16, a.k_msb + r * DH + sub * 16);
    if (LSB) cp_async8(wsm + SM::kLsb + (s * 32 + lane) * 8, a.k_lsb + r * (DH / 2) + sub * 8);
  }
  cp_async_commit();
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    if (rid[s] < 0) continue;
    const int64_t r = plane0 + rid[s];
    cp_async16(wsm + SM::vMsb + (s * 32 + lane) * 16, a.v_msb + r * DH + sub * 16);
    if (LSB) cp_async8(wsm + SM::vLsb + (s * 32 + lane) * 8, a.v_lsb + r * (DH / 2) + sub * 8);
  }
  cp_async_commit();
  const float c1 = 16.0f * ks * a.sm_scale, c2 = ks * a.sm_scale;

  // ---- scores of both variants -----------------------------------------------------------------
  cp_async_wait<1>();
  float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll 4
  for (int s = 0; s < STEPS; ++s) {
    // d1 = q . MSB_j; d2 = q . LSB_j; the full-precision dot product is 16 d1 + d2
    const uint4 km = *reinterpret_cast<const uint4*>(wsm + SM::kMsb + (s * 32 + lane) * 16);
    float2 f[8];
    msb16(km, f);
    float2 a1 = make_float2(0.0f, 0.0f), a2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) a1 = ffma2(qf[i], f[i], a1);
    if (LSB) {
      const uint2 kl = *reinterpret_cast<const uint2*>(wsm + SM::kLsb + (s * 32 + lane) * 8);
      float2 g[8];
      lsb16(kl, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) a2 = ffma2(qf[i], g[i], a2);
    }
    float d1 = a1.x + a1.y, d2 = a2.x + a2.y;
#pragma unroll
    for (int o2 = 1; o2 < LPK; o2 <<= 1) {
      d1 += __shfl_xor_sync(0xffffffffu, d1, o2);
      if (LSB) d2 += __shfl_xor_sync(0xffffffffu, d2, o2);
    }
    if ((valid >> s) & 1u) {   // a slice past the key list was not copied: its value is not used
      const float s1 = d1 * c1, s2 = fmaf(16.0f, d1, d2) * c2;
      m1 = fmaxf(m1, s1);
      if (LSB) m2 = fmaxf(m2, s2);
      if (sub == 0) {
        s_sc[s * KPW + grp] = s1;
        if (LSB) s_sc[(NV - 1) * ITEM + s * KPW + grp] = s2;
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
      const float e1 = expf(s_sc[k] - m1);
      s_sc[k] = e1;
      e_out[j] = e1;
      l1 += e1;
      if (LSB) {
        const float e2 = expf(s_sc[(NV - 1) * ITEM + k] - m2);
        s_sc[(NV - 1) * ITEM + k] = e2;
        e_out[vstride + j] = e2;
        l2 += e2;
      }
    }
  }
  l1 = warp_sum(l1);
  if (LSB) l2 = warp_sum(l2);
  __syncwarp();

  // ---- sums of e * V codes ----------------------------------------------------------------------
  cp_async_wait<0>();
  float2 o1[8], o2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o1[i] = o2[i] = make_float2(0.0f, 0.0f);
#pragma unroll 4
  for (int s = 0; s < STEPS; ++s) {
    if (!((valid >> s) & 1u)) continue;
    const int k = s * KPW + grp;
    const uint4 vm = *reinterpret_cast<const uint4*>(wsm + SM::vMsb + (s * 32 + lane) * 16);
    float2 f[8];
    msb16(vm, f);
    const float e1 = s_sc[k];
    const float2 e1v = make_float2(e1, e1);
#pragma unroll
    for (int i = 0; i < 8; ++i) o1[i] = ffma2(e1v, f[i], o1[i]);
    if (LSB) {
      const uint2 vl = *reinterpret_cast<const uint2*>(wsm + SM::vLsb + (s * 32 + lane) * 8);
      float2 g[8];
      lsb16(vl, g);
      const float e2 = s_sc[(NV - 1) * ITEM + k];
      const float2 e2v = make_float2(e2, e2), sixteen = make_float2(16.0f, 16.0f);
#pragma unroll
      for (int i = 0; i < 8; ++i) o2[i] = ffma2(e2v, ffma2(sixteen, f[i], g[i]), o2[i]);
    }
  }
  // add the lane groups' sums through shared memory (the K MSB area, read by every lane before
  // the last warp barrier), in group order
  float* s_o = reinterpret_cast<float*>(wsm + SM::kMsb);   // [KPW][NV * DH]
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_o[grp * NV * DH + sub * 16 + 2 * i] = o1[i].x;
    s_o[grp * NV * DH + sub * 16 + 2 * i + 1] = o1[i].y;
    if (LSB) {
      s_o[grp * NV * DH + DH + sub * 16 + 2 * i] = o2[i].x;
      s_o[grp * NV * DH + DH + sub * 16 + 2 * i + 1] = o2[i].y;
    }
  }
  __syncwarp();
  float* o_out = p.dec_o + (bs * p.dec_items + item) * 2 * DH;
  for (int t = lane; t < NV * DH; t += 32) {
    float v = 0.0f;
#pragma unroll
    for (int g = 0; g < KPW; ++g) v += s_o[g * NV * DH + t];
    o_out[t] = v;
  }
  if (lane == 0)
    reinterpret_cast<float4*>(p.dec_stat)[bs * p.dec_items + item] = make_float4(m1, l1, LSB ? m2 : m1, LSB ? l2 : l1);
}

// Row statistics of one kept head folded by one warp in a fixed order (lane-strided item partials,
// then a butterfly); returns whether the row refetches, and the chosen variant's (m, 1/ell).
// v0: this lane's first item statistics, st[lane] (kNoItem past the row), loaded by the caller so
// that the load can be in flight with others.
__device__ __forceinline__ float4 no_item() { return make_float4(-INFINITY, 0.0f, -INFINITY, 0.0f); }
__device__ __forceinline__ float4 first_item(const float4* st, int NI) {
  const int lane = threadIdx.x & 31;
  return lane < NI ? st[lane] : no_item();
}
template <bool LSB>
__device__ __forceinline__ bool fold_row(float4 v0, const float4* st, int NI, float theta, float* m_out,
                                         float* inv_l_out) {
  const int lane = threadIdx.x & 31;
  float M1 = v0.x, M2 = v0.z;
  for (int i = lane + 32; i < NI; i += 32) {
    const float4 v = st[i];
    M1 = fmaxf(M1, v.x);
    M2 = fmaxf(M2, v.z);
  }
  M1 = warp_max(M1);
  if (LSB) M2 = warp_max(M2);
  float L1 = 0.0f, L2 = 0.0f;
  if (lane < NI) {
    L1 = v0.y * expf(v0.x - M1);
    if (LSB) L2 = v0.w * expf(v0.z - M2);
  }
  for (int i = lane + 32; i < NI; i += 32) {
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
template <bool LSB>
__device__ __forceinline__ bool fold_row(const float4* st, int NI, float theta, float* m_out, float* inv_l_out) {
  return fold_row<LSB>(first_item(st, NI), st, NI, theta, m_out, inv_l_out);
}

constexpr int kCWarps = kCThreads / 32;
constexpr int kCSlots = 4;    // kept heads per warp whose statistics a token block loads up front
constexpr int kCHeads = 16;   // kept heads whose exponentials a token-block thread loads up front
constexpr int kCItems = 4;    // items per thread whose partial outputs an output block loads up front

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
    const int j = j0 + threadIdx.x;
    const bool jv = j < n;
    const int64_t vstride = static_cast<int64_t>(a.B) * HK * n;
    const float* e = p.dec_e + static_cast<int64_t>(b) * HK * n + j;
    // independent of the row statistics, so in flight with their loads: the key's importance
    // entry and the exponentials of both variants for the first kCHeads kept heads
    int64_t dst = 0;
    float cur = 0.0f;
    if (jv && a.tok_imp) {
      const int64_t col = a.tok_imp_map ? a.tok_imp_map[static_cast<int64_t>(b) * a.tok_imp_map_ld + j] : j;
      dst = static_cast<int64_t>(b) * a.tok_imp_ld + col;
      cur = a.tok_imp[dst];
    }
    float e1[kCHeads], e2[kCHeads];
#pragma unroll
    for (int u = 0; u < kCHeads; ++u) {
      e1[u] = jv && u < HK ? e[static_cast<int64_t>(u) * n] : 0.0f;
      e2[u] = LSB && jv && u < HK ? e[vstride + static_cast<int64_t>(u) * n] : 0.0f;
    }
    float* factor = sh;                                   // [HK][TI] factors of items it0 ..
    int* use_full = reinterpret_cast<int*>(sh + HK * TI); // [HK]
    float4 pre[kCSlots];
#pragma unroll
    for (int u = 0; u < kCSlots; ++u) {
      const int slot = warp + u * kCWarps;
      pre[u] = slot < HK ? first_item(stats + static_cast<int64_t>(slot) * NI, NI) : no_item();
    }
    auto fold_slot = [&](int slot, float4 v0) {
      const float4* st = stats + static_cast<int64_t>(slot) * NI;
      float m, inv_l;
      const bool full = fold_row<LSB>(v0, st, NI, a.refetch_threshold, &m, &inv_l);
      // the factors of items it0 .. it0 + TI - 1: from the first-item registers when they hold them
      float4 v;
      if (it0 + TI <= 32) {
        v.x = __shfl_sync(0xffffffffu, v0.x, (it0 + lane) & 31);
        v.z = __shfl_sync(0xffffffffu, v0.z, (it0 + lane) & 31);
      } else if (lane < TI && it0 + lane < NI) {
        v = st[it0 + lane];
      }
      if (lane < TI && it0 + lane < NI) factor[slot * TI + lane] = expf((full ? v.z : v.x) - m) * inv_l;
      if (lane == 0) use_full[slot] = full ? 1 : 0;
    };
#pragma unroll
    for (int u = 0; u < kCSlots; ++u)
      if (warp + u * kCWarps < HK) fold_slot(warp + u * kCWarps, pre[u]);
    for (int slot = warp + kCSlots * kCWarps; slot < HK; slot += kCWarps)
      fold_slot(slot, first_item(stats + static_cast<int64_t>(slot) * NI, NI));
    __syncthreads();
    if (!jv) return;
    const int it = j / ITEM - it0;
    float t = 0.0f;
    float* hc = p.head_col ? p.head_col + static_cast<int64_t>(b) * HK * n + j : nullptr;
#pragma unroll
    for (int u = 0; u < kCHeads; ++u) {
      if (u < HK) {
        const float pj = (use_full[u] ? e2[u] : e1[u]) * factor[u * TI + it];
        t += pj;
        if (hc) hc[static_cast<int64_t>(u) * n] = pj;
      }
    }
    for (int slot = kCHeads; slot < HK; ++slot) {
      const float pj = e[(use_full[slot] ? vstride : 0) + static_cast<int64_t>(slot) * n] * factor[slot * TI + it];
      t += pj;
      if (hc) hc[static_cast<int64_t>(slot) * n] = pj;
    }
    if (a.tok_imp) a.tok_imp[dst] = cur + t;
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
  const int64_t bhh = static_cast<int64_t>(b) * a.H + h;
  const float4* st = stats + static_cast<int64_t>(slot) * NI;
  const int dim = threadIdx.x % DH, g = threadIdx.x / DH;
  // everything this thread reads, issued before the fold: the row's first item statistics, this
  // thread's items' statistics and partial outputs of both variants, the value scale
  const float4 v0 = first_item(st, NI);
  const float* op = p.dec_o + (static_cast<int64_t>(b) * HK + slot) * NI * 2 * DH + dim;
  float2 sx[kCItems];
  float o1[kCItems], o2[kCItems];
#pragma unroll
  for (int u = 0; u < kCItems; ++u) {
    const int i = g + u * IG;
    const bool iv = i < NI;
    const float4 si = iv ? st[i] : no_item();
    sx[u] = make_float2(si.x, si.z);
    o1[u] = iv ? op[static_cast<int64_t>(i) * 2 * DH] : 0.0f;
    o2[u] = LSB && iv ? op[static_cast<int64_t>(i) * 2 * DH + DH] : 0.0f;
  }
  const float vs = a.v_scale[bhh];
  // every warp folds the row (the same loads and order, so the same decision in every warp)
  float m, inv_l;
  const bool full = fold_row<LSB>(v0, st, NI, a.refetch_threshold, &m, &inv_l);
  {
    float v = 0.0f;
#pragma unroll
    for (int u = 0; u < kCItems; ++u)
      if (g + u * IG < NI) v += (full ? o2[u] : o1[u]) * (expf((full ? sx[u].y : sx[u].x) - m) * inv_l);
    for (int i = g + kCItems * IG; i < NI; i += IG) {
      const float4 si = st[i];
      v += op[static_cast<int64_t>(i) * 2 * DH + (full ? DH : 0)] * (expf((full ? si.z : si.x) - m) * inv_l);
    }
    part[g][dim] = v;
  }
  __syncthreads();
  float absv = 0.0f;
  if (static_cast<int>(threadIdx.x) < DH) {
    float v = 0.0f;
#pragma unroll
    for (int gg = 0; gg < IG; ++gg) v += part[gg][threadIdx.x];
    // the MSB-pass sums hold e * MSB_j; its dequantized value is s_v * 16 * MSB_j
    v *= vs * (full ? 1.0f : 16.0f);
    st_from_float(o + threadIdx.x, v);
    absv = fabsf(v);
  }
  absv = warp_sum(absv);
  if (lane == 0) red[warp] = absv;
  __syncthreads();
  if (threadIdx.x == 0) {
    float hs = 0.0f;
    for (int w = 0; w < DH / 32; ++w) hs += red[w];
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

// Predicated form: the refetch decision of every (sequence, kept head) row from its MSB-pass item
// statistics, folded exactly as the combine step folds them (one warp per row).
__global__ void __launch_bounds__(32) attn_decode_flag_kernel(AttnProblem p) {
  const int slot = blockIdx.x, b = blockIdx.y;
  const int64_t row = static_cast<int64_t>(b) * p.a.H_kept + slot;
  float m, inv_l;
  // the MSB pass wrote (m1, l1, m1, l1): the full-precision fold sees the MSB statistics
  const bool full = fold_row<true>(reinterpret_cast<const float4*>(p.dec_stat) + row * p.dec_items, p.dec_items,
                                   p.a.refetch_threshold, &m, &inv_l);
  if (threadIdx.x == 0) p.dec_flag[row] = full ? 1 : 0;
}

// dynamic shared memory of the combine kernel: a token block's factor table and flags
size_t combine_smem(int d_h, int H_kept) {
  const int item_rows = d_h == 64 ? DGeom<64>::ITEM : DGeom<128>::ITEM;
  const int ti = (kCThreads + item_rows - 1) / item_rows + 1;
  return static_cast<size_t>(H_kept) * (ti + 1) * 4;
}

template <int DH, typename QT, bool LSB, bool FLAGGED>
int32_t launch_items(const AttnProblem& p, cudaStream_t st) {
  constexpr int smem = kDWarps * DSmem<DH, LSB>::bytes;
  static DeviceOnce once;
  int dev = 0;
  SPT_TRY(once_per_device(once, &dev, [](int) -> int32_t {
    SPT_CUDA(cudaFuncSetAttribute(attn_decode_items_kernel<DH, QT, LSB, FLAGGED>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    return SPATTEN_OK;
  }));
  const int64_t per_seq = static_cast<int64_t>(p.dec_items) * p.a.H_kept;
  attn_decode_items_kernel<DH, QT, LSB, FLAGGED>
      <<<dim3(static_cast<unsigned>(ceil_div(per_seq, kDWarps)), p.a.B), kDWarps * 32, smem, st>>>(p);
  return launch_status();
}

template <int DH, typename QT, bool LSB>
int32_t launch(const AttnProblem& p, cudaStream_t st) {
  if (LSB && p.dec_flag) {
    // predicated: the MSB planes for every row, the decision, the LSB planes for the flagged rows
    SPT_TRY((launch_items<DH, QT, false, false>(p, st)));
    attn_decode_flag_kernel<<<dim3(p.a.H_kept, p.a.B), 32, 0, st>>>(p);
    SPT_TRY(launch_status());
    SPT_TRY((launch_items<DH, QT, true, true>(p, st)));
  } else {
    SPT_TRY((launch_items<DH, QT, LSB, false>(p, st)));
  }
  const int nblk = static_cast<int>(ceil_div(p.a.n_kv, kCThreads));
  const int slots = p.a.H_kept + (p.a.zero_pruned_heads ? p.a.H - p.a.H_kept : 0);
  attn_decode_combine_kernel<DH, QT, LSB>
      <<<dim3(nblk + slots, p.a.B), kCThreads, combine_smem(DH, p.a.H_kept), st>>>(p);
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
  // up to 12 K items per row; a token block of the combine step keeps every kept head's factors
  // in shared memory (48 KB without opting in)
  const int64_t items = ceil_div(a.n_kv, decode_item_rows(a.d_h));
  return items <= 12 * 1024 && combine_smem(a.d_h, a.H_kept) <= 48 * 1024;
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
