// K2: prefill attention with importance on the 5th-generation tensor cores (tcgen05 + TMEM),
// warp-specialized and pipelined.
//
// SpAtten §II "Attention mechanism" (S = Q K^T scaled, row softmax, P V), §II "Cascade pruning"
// (token importance = column sums of P; head importance = sum |O|), §IV.E "Progressive
// Quantization" (MSB pass; rows whose max probability is below the threshold are recomputed with
// the LSBs).  One CTA = (sequence, kept head, 128 query rows).
//
// Exact operands: K and V are 12-bit codes q = 16*MSB + LSB; 16*MSB (8 significant bits) and
// LSB (0..15) are exact in bf16, so the MMAs see the codes unrounded and the scales multiply the
// float32 accumulators:
//   S_msb = s_k * sm * (Q . (16 MSB)^T),   S_full = S_msb + s_k * sm * (Q . LSB^T)
//   O     = s_v * (P . 16 MSB_v  [+ P . LSB_v for refetched rows])
// The LSB products land in their own TMEM columns; each softmax thread adds them only for its own
// row when that row refetches, so no masked operand copies are needed.
//
// Roles (256 threads):
//   warps 0-3  softmax: thread i owns query row i = TMEM lane i (warp w reads lane quadrant w)
//   warps 4-6  producers: load Q once, dequantize K/V code tiles into 2-stage shared rings
//   warp 7     MMA issue (lane 0) and TMEM allocation
// Key tiles hold 16 KB of bf16 codes: 128 keys at d_h = 64, 64 keys at d_h = 128.
// Passes over the keys (all pipelined through mbarriers; every wait is bounded):
//   A   S_msb tiles (double-buffered in TMEM) -> online row max / exp-sum -> refetch flags
//   A'  only if some row is flagged: S and C = Q.LSB^T (single-buffered) -> stats of flagged rows
//   B   S (+C) -> P = exp(S - m)/ell in float32 -> column sums by a 31-shuffle butterfly
//       (deterministic) -> P in bf16 to shared memory (double-buffered) -> O += P V (+ O_lsb)
//       with QK of tile t+1 issued before PV of tile t
// Operand layouts: UMMA 128-byte swizzle; Q, K, P K-major; V MN-major (plain key rows).
// TMEM (512 columns): S buffers [0, 2*KT), O [2*KT, 2*KT + d_h), O_lsb after it; in refetch mode
// S uses buffer 0 and C buffer 1.
#include "attention.cuh"
#include "tc_ptx.cuh"

namespace spt {
namespace {

using namespace tc;

constexpr int kThreads = 256;
constexpr int kSoftmaxThreads = 128;
constexpr int kProducerThreads = 96;
constexpr int kMmaWarp = 7;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 26;   // polls of one mbarrier phase before giving up
constexpr float kLog2e = 1.4426950408889634f;

template <int DH>
struct Cfg {
  static constexpr int KT = DH == 64 ? 128 : 64;            // keys per tile
  static constexpr uint32_t QB = 128u * DH * 2u;             // Q tile bytes
  static constexpr uint32_t TB = static_cast<uint32_t>(KT) * DH * 2u;   // K or V tile (16 KB)
  static constexpr uint32_t PB = 128u * KT * 2u;             // P tile bytes
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + QB;                    // 2 stages
  static constexpr uint32_t oKL = oK + 2 * TB;
  static constexpr uint32_t oV = oKL + 2 * TB;
  static constexpr uint32_t oVL = oV + 2 * TB;
  static constexpr uint32_t oP = oVL + 2 * TB;               // 2 buffers
  static constexpr uint32_t kEnd = oP + 2 * PB;
  static constexpr uint32_t kSmem = kEnd + 1024u;
  static constexpr uint32_t tS = 0;                          // TMEM column offsets
  static constexpr uint32_t tO = 2u * KT;
  static constexpr uint32_t tO2 = 2u * KT + DH;
  static constexpr int CH = KT / 32;                         // 32-column chunks per tile
};

// barrier slots
enum : int {
  B_Q = 0,
  B_KFULL = 1,    // +stage (2)
  B_KEMPTY = 3,   // +stage
  B_VFULL = 5,    // +stage
  B_VEMPTY = 7,   // +stage
  B_SFULL = 9,    // +buffer
  B_SFREE = 11,   // +buffer
  B_PFULL = 13,   // +buffer
  B_PFREE = 15,   // +buffer
  B_ODONE = 17,
  B_COUNT = 18
};

// byte offset of 16-byte chunk c8 of `row` in a tile whose 64-element column blocks each hold
// `rows` rows of 128 bytes (128-byte swizzle)
__device__ __forceinline__ uint32_t tile_off(uint32_t row, uint32_t c8, uint32_t rows) {
  return (c8 >> 3) * rows * 128u + sw128_offset(row, c8 & 7u);
}

__device__ __forceinline__ void cvt16_s8x16(uint4 raw, uint32_t* out8) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float f0 = 16.0f * static_cast<float>(static_cast<int8_t>(w[i] & 0xFFu));
    const float f1 = 16.0f * static_cast<float>(static_cast<int8_t>((w[i] >> 8) & 0xFFu));
    const float f2 = 16.0f * static_cast<float>(static_cast<int8_t>((w[i] >> 16) & 0xFFu));
    const float f3 = 16.0f * static_cast<float>(static_cast<int8_t>(w[i] >> 24));
    out8[2 * i] = pack_bf16x2(f0, f1);
    out8[2 * i + 1] = pack_bf16x2(f2, f3);
  }
}
__device__ __forceinline__ void cvt_u4x16(uint2 raw, uint32_t* out8) {
  const uint32_t w[2] = {raw.x, raw.y};
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      out8[4 * i + k] = pack_bf16x2(static_cast<float>((w[i] >> (8 * k)) & 0xFu),
                                    static_cast<float>((w[i] >> (8 * k + 4)) & 0xFu));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_sync_softmax() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// bounded wait that also gives up once another role has aborted
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

// column sums over the 32 rows of a warp: afterwards lane l holds the sum of column l
__device__ __forceinline__ float warp_colsum32(float* v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = upper ? v[j] : v[j + off];
      const float keep = upper ? v[j + off] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

enum Pass { kPassA = 0, kPassA2 = 1, kPassB = 2 };

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(AttnProblem p) {
  using C = Cfg<DH>;
  constexpr int KT = C::KT;
  const spatten_attn_args& a = p.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bars[B_COUNT];
  __shared__ uint32_t tmem_base_s;
  __shared__ float colred[2][4][KT];
  __shared__ float hred[4];
  __shared__ int abort_s;

  const int qt = blockIdx.x, slot = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = qt * 128;
  const int h = head_of_slot(a, b, slot);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);

  if (slot >= a.H_kept) {   // pruned head: zero its output rows (no TMEM, no barrier)
    if (h < 0) return;
    for (int e = tid; e < 128 * (DH / 8); e += kThreads) {
      const int i = i0 + e / (DH / 8), c8 = e % (DH / 8);
      if (i < a.n_q)
        *reinterpret_cast<uint4*>(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok +
                                  static_cast<int64_t>(h) * DH + c8 * 8) = make_uint4(0, 0, 0, 0);
    }
    return;
  }

  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_s, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    abort_s = 0;
    mbar_init(&bars[B_Q], kProducerThreads);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_KFULL + s], kProducerThreads);
      mbar_init(&bars[B_VFULL + s], kProducerThreads);
      mbar_init(&bars[B_KEMPTY + s], 1);
      mbar_init(&bars[B_VEMPTY + s], 1);
      mbar_init(&bars[B_SFULL + s], 1);
      mbar_init(&bars[B_SFREE + s], kSoftmaxThreads);
      mbar_init(&bars[B_PFULL + s], kSoftmaxThreads);
      mbar_init(&bars[B_PFREE + s], 1);
    }
    mbar_init(&bars[B_ODONE], 1);
    fence_mbar_init();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;

  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t plane0 = bh * a.kv_cap;
  const int32_t* kv_idx = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;
  const int n_tiles = (a.n_kv + KT - 1) / KT;
  const uint32_t sQ = smem_u32(smem + C::oQ);

  // ---------------------------------------------------------------------------------------------
  // role state (each role only touches its own)
  // ---------------------------------------------------------------------------------------------
  uint32_t kc = 0, vc = 0;          // K / V ring uses (producer and MMA)
  uint32_t sc[2] = {0, 0};          // S buffer uses (MMA and softmax)
  uint32_t pc[2] = {0, 0};          // P buffer uses (MMA and softmax)
  bool aborted = false;

  // softmax row state
  const int row = tid, i = i0 + row;
  const bool row_ok = tid < 128 && i < a.n_q;
  float m2 = -INFINITY, l = 0.0f;
  bool flag = false;

  // ---- producers: dequantize one code tile -----------------------------------------------------
  auto produce = [&](int t, const int8_t* msb, const uint8_t* lsb, uint32_t off_hi, uint32_t off_lo) {
    const int ptid = tid - 128;
    constexpr int L16 = DH / 16;
    for (int e = ptid; e < KT * L16; e += kProducerThreads) {
      const int r = e / L16, c16 = e % L16;
      const int key = t * KT + r;
      uint32_t hi[8], lo[8];
      if (key < a.n_kv) {
        const int64_t prow = plane0 + (kv_idx ? kv_idx[key] : key);
        cvt16_s8x16(__ldg(reinterpret_cast<const uint4*>(msb + prow * DH) + c16), hi);
        if (lsb) cvt_u4x16(__ldg(reinterpret_cast<const uint2*>(lsb + prow * (DH / 2)) + c16), lo);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) hi[q] = lo[q] = 0u;
      }
      *reinterpret_cast<uint4*>(smem + off_hi + tile_off(r, 2 * c16, KT)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + off_hi + tile_off(r, 2 * c16 + 1, KT)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
      if (lsb) {
        *reinterpret_cast<uint4*>(smem + off_lo + tile_off(r, 2 * c16, KT)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4*>(smem + off_lo + tile_off(r, 2 * c16 + 1, KT)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
      }
    }
    fence_async_smem();
  };

  auto run_producer = [&](int pass, bool refetch) {
    for (int t = 0; t < n_tiles && !aborted; ++t) {
      const uint32_t ks = kc & 1u;
      if (!wait_bar(&bars[B_KEMPTY + ks], ((kc >> 1) & 1u) ^ 1u, abort_flag)) { aborted = true; break; }
      produce(t, a.k_msb, refetch ? a.k_lsb : nullptr, C::oK + ks * C::TB, C::oKL + ks * C::TB);
      mbar_arrive(&bars[B_KFULL + ks]);
      ++kc;
      if (pass == kPassB) {
        const uint32_t vs = vc & 1u;
        if (!wait_bar(&bars[B_VEMPTY + vs], ((vc >> 1) & 1u) ^ 1u, abort_flag)) { aborted = true; break; }
        produce(t, a.v_msb, refetch ? a.v_lsb : nullptr, C::oV + vs * C::TB, C::oVL + vs * C::TB);
        mbar_arrive(&bars[B_VFULL + vs]);
        ++vc;
      }
    }
  };

  // ---- MMA issue ---------------------------------------------------------------------------------
  constexpr uint32_t kIdQK = idesc_bf16(128, KT, false, false);
  constexpr uint32_t kIdPV = idesc_bf16(128, DH, false, true);
  auto issue_qk = [&](int t, bool refetch) -> bool {
    const uint32_t ks = kc & 1u;
    if (!wait_bar(&bars[B_KFULL + ks], (kc >> 1) & 1u, abort_flag)) return false;
    const int sb = refetch ? 0 : (t & 1);
    if (!wait_bar(&bars[B_SFREE + sb], (sc[sb] & 1u) ^ 1u, abort_flag)) return false;
    tc_after_sync();
    const uint32_t sK = smem_u32(smem + C::oK + ks * C::TB), sKL = smem_u32(smem + C::oKL + ks * C::TB);
    const uint32_t dS = tmem + C::tS + sb * KT, dC = tmem + C::tS + KT;
#pragma unroll
    for (int s = 0; s < DH / 16; ++s) {
      const uint32_t qoff = (s >> 2) * 16384u + (s & 3) * 32u;
      const uint32_t koff = (s >> 2) * (KT * 128u) + (s & 3) * 32u;
      mma_bf16(dS, desc_sw128(sQ + qoff, 16, 1024), desc_sw128(sK + koff, 16, 1024), kIdQK, s > 0);
    }
    if (refetch) {
#pragma unroll
      for (int s = 0; s < DH / 16; ++s) {
        const uint32_t qoff = (s >> 2) * 16384u + (s & 3) * 32u;
        const uint32_t koff = (s >> 2) * (KT * 128u) + (s & 3) * 32u;
        mma_bf16(dC, desc_sw128(sQ + qoff, 16, 1024), desc_sw128(sKL + koff, 16, 1024), kIdQK, s > 0);
      }
    }
    mma_commit(&bars[B_SFULL + sb]);
    mma_commit(&bars[B_KEMPTY + ks]);
    ++sc[sb];
    ++kc;
    return true;
  };
  auto issue_pv = [&](int t, bool refetch) -> bool {
    const int pb = t & 1;
    if (!wait_bar(&bars[B_PFULL + pb], pc[pb] & 1u, abort_flag)) return false;
    const uint32_t vs = vc & 1u;
    if (!wait_bar(&bars[B_VFULL + vs], (vc >> 1) & 1u, abort_flag)) return false;
    tc_after_sync();
    const uint32_t sP = smem_u32(smem + C::oP + pb * C::PB);
    const uint32_t sV = smem_u32(smem + C::oV + vs * C::TB), sVL = smem_u32(smem + C::oVL + vs * C::TB);
#pragma unroll
    for (int s = 0; s < KT / 16; ++s) {
      const uint32_t poff = (s >> 2) * 16384u + (s & 3) * 32u;
      const uint32_t voff = s * 2048u;
      const uint32_t acc = (t > 0 || s > 0) ? 1u : 0u;
      mma_bf16(tmem + C::tO, desc_sw128(sP + poff, 16, 1024), desc_sw128(sV + voff, KT * 128u, 1024), kIdPV, acc);
      if (refetch)
        mma_bf16(tmem + C::tO2, desc_sw128(sP + poff, 16, 1024), desc_sw128(sVL + voff, KT * 128u, 1024), kIdPV, acc);
    }
    mma_commit(&bars[B_PFREE + pb]);
    mma_commit(&bars[B_VEMPTY + vs]);
    ++pc[pb];
    ++vc;
    return true;
  };
  auto run_mma = [&](int pass, bool refetch) {
    if (lane != 0) return;
    if (pass != kPassB) {
      for (int t = 0; t < n_tiles; ++t)
        if (!issue_qk(t, refetch)) { aborted = true; return; }
      return;
    }
    if (!issue_qk(0, refetch)) { aborted = true; return; }
    for (int t = 0; t < n_tiles; ++t) {
      if (t + 1 < n_tiles && !issue_qk(t + 1, refetch)) { aborted = true; return; }
      if (!issue_pv(t, refetch)) { aborted = true; return; }
    }
    mma_commit(&bars[B_ODONE]);
  };

  // ---- softmax ------------------------------------------------------------------------------------
  const float c2 = a.k_scale[bh] * a.sm_scale * kLog2e;   // raw accumulator -> log2-domain score
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  auto run_stats = [&](bool refetch) {   // pass A (refetch = false) or A' (refetch = true)
    float mx2 = -INFINITY, lx = 0.0f;
    for (int t = 0; t < n_tiles; ++t) {
      const int sb = refetch ? 0 : (t & 1);
      if (!wait_bar(&bars[B_SFULL + sb], sc[sb] & 1u, abort_flag)) { aborted = true; break; }
      tc_after_sync();
#pragma unroll 1
      for (int ch = 0; ch < C::CH; ++ch) {
        float v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_base + C::tS + sb * KT + ch * 32, v);
        if (refetch) {
          float w[32];
          tmem_ld32(tmem + lane_base + C::tS + KT + ch * 32, w);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += w[j];
        } else {
          tmem_ld_wait();
        }
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = (t * KT + ch * 32 + j < a.n_kv) ? v[j] * c2 : -INFINITY;
          mx = fmaxf(mx, v[j]);
        }
        if (mx != -INFINITY) {
          const float mn = fmaxf(mx2, mx);
          float add = 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) add += ex2(v[j] - mn);
          lx = lx * ex2(mx2 - mn) + add;
          mx2 = mn;
        }
      }
      tc_before_sync();
      mbar_arrive(&bars[B_SFREE + sb]);
      ++sc[sb];
    }
    if (!refetch) {
      m2 = mx2;
      l = lx;
    } else if (flag) {
      m2 = mx2;
      l = lx;
    }
  };

  const int64_t part_row = ((static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt) * a.n_kv;
  auto run_probs = [&](bool refetch) {   // pass B
    const float inv_l = 1.0f / l;
    for (int t = 0; t < n_tiles; ++t) {
      const int sb = refetch ? 0 : (t & 1);
      const int pb = t & 1;
      if (!wait_bar(&bars[B_PFREE + pb], (pc[pb] & 1u) ^ 1u, abort_flag)) { aborted = true; break; }
      if (!wait_bar(&bars[B_SFULL + sb], sc[sb] & 1u, abort_flag)) { aborted = true; break; }
      tc_after_sync();
      uint8_t* Pt = smem + C::oP + pb * C::PB;
#pragma unroll 1
      for (int ch = 0; ch < C::CH; ++ch) {
        float v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_base + C::tS + sb * KT + ch * 32, v);
        if (refetch) {
          float w[32];
          tmem_ld32(tmem + lane_base + C::tS + KT + ch * 32, w);
          tmem_ld_wait();
          if (flag) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += w[j];
          }
        } else {
          tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const bool ok = row_ok && (t * KT + ch * 32 + j < a.n_kv);
          v[j] = ok ? ex2(v[j] * c2 - m2) * inv_l : 0.0f;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t c8 = ch * 4 + q4;
          *reinterpret_cast<uint4*>(Pt + tile_off(row, c8, 128)) =
              make_uint4(pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]), pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                         pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
        }
        colred[t & 1][warp][ch * 32 + lane] = warp_colsum32(v);
      }
      tc_before_sync();
      mbar_arrive(&bars[B_SFREE + sb]);
      ++sc[sb];
      fence_async_smem();
      mbar_arrive(&bars[B_PFULL + pb]);
      ++pc[pb];
      named_sync_softmax();
      for (int kk = tid; kk < KT; kk += kSoftmaxThreads) {
        const int key = t * KT + kk;
        if (key < a.n_kv)
          p.tok_part[part_row + key] =
              ((colred[t & 1][0][kk] + colred[t & 1][1][kk]) + colred[t & 1][2][kk]) + colred[t & 1][3][kk];
      }
    }
  };

  // ---------------------------------------------------------------------------------------------
  // producers load Q once
  // ---------------------------------------------------------------------------------------------
  if (warp >= 4 && warp < kMmaWarp) {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
    for (int e = tid - 128; e < 128 * (DH / 8); e += kProducerThreads) {
      const int r = e / (DH / 8), c8 = e % (DH / 8), qi = i0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (qi < a.n_q)
        v = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * a.n_q + qi) * a.q_ld_tok +
                                                 static_cast<int64_t>(h) * DH) + c8);
      *reinterpret_cast<uint4*>(smem + C::oQ + tile_off(r, c8, 128)) = v;
    }
    fence_async_smem();
    mbar_arrive(&bars[B_Q]);
  } else if (warp == kMmaWarp && lane == 0) {
    if (!wait_bar(&bars[B_Q], 0, abort_flag)) aborted = true;
  }

  // ---- pass A ----------------------------------------------------------------------------------
  if (!aborted) {
    if (warp < 4) run_stats(false);
    else if (warp < kMmaWarp) run_producer(kPassA, false);
    else run_mma(kPassA, false);
  }
  if (warp < 4) flag = !aborted && a.quantized && row_ok && (1.0f / l < a.refetch_threshold);
  const bool any_flag = __syncthreads_or(flag) != 0;
  if (__syncthreads_or(aborted)) aborted = true;

  // ---- pass A' ---------------------------------------------------------------------------------
  if (any_flag && !aborted) {
    if (warp < 4) run_stats(true);
    else if (warp < kMmaWarp) run_producer(kPassA2, true);
    else run_mma(kPassA2, true);
  }
  if (__syncthreads_or(aborted)) aborted = true;

  // ---- pass B ----------------------------------------------------------------------------------
  if (!aborted) {
    if (warp < 4) run_probs(any_flag);
    else if (warp < kMmaWarp) run_producer(kPassB, any_flag);
    else run_mma(kPassB, any_flag);
  }

  // ---- epilogue (softmax warps): O, head importance, flags ----------------------------------------
  float habs = 0.0f;
  if (warp < 4 && !aborted) {
    if (!wait_bar(&bars[B_ODONE], 0, abort_flag)) aborted = true;
    tc_after_sync();
    if (!aborted) {
      const float vs = a.v_scale[bh];
#pragma unroll 1
      for (int ch = 0; ch < DH / 32; ++ch) {
        float v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_base + C::tO + ch * 32, v);
        if (any_flag) {
          float w[32];
          tmem_ld32(tmem + lane_base + C::tO2 + ch * 32, w);
          tmem_ld_wait();
          if (flag) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += w[j];
          }
        } else {
          tmem_ld_wait();
        }
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float x0 = v[2 * j] * vs, x1 = v[2 * j + 1] * vs;
            habs += fabsf(x0) + fabsf(x1);
            pk[j] = pack_bf16x2(x0, x1);
          }
          uint4* dst = reinterpret_cast<uint4*>(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok +
                                                static_cast<int64_t>(h) * DH + ch * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      if (row_ok && a.refetch_flags) a.refetch_flags[bh * a.refetch_flags_ld + i] = flag ? 1 : 0;
    }
  }
  if (warp < 4) {
    habs = warp_sum(habs);
    if (lane == 0) hred[warp] = habs;
  }
  const int nflag = __syncthreads_count(flag);
  if (__syncthreads_or(aborted)) aborted = true;
  tc_before_sync();
  __syncthreads();
  if (tid == 0) {
    p.head_part[(static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt] = ((hred[0] + hred[1]) + hred[2]) + hred[3];
    if (nflag && a.refetch_count) atomicAdd(a.refetch_count, nflag);
    if (aborted) report(a.dev_status, SPATTEN_E_TIMEOUT);
  }
  if (warp == kMmaWarp) {
    tc_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DH>
int32_t launch(const AttnProblem& p, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    SPT_CUDA(cudaFuncSetAttribute(attn_tc_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(Cfg<DH>::kSmem)));
    configured[dev] = true;
  }
  const int slots = p.a.H_kept + (p.a.zero_pruned_heads ? p.a.H - p.a.H_kept : 0);
  attn_tc_kernel<DH><<<dim3(p.n_qt, slots, p.a.B), kThreads, Cfg<DH>::kSmem, st>>>(p);
  return launch_status();
}

}  // namespace

bool attn_tc_supported(const spatten_attn_args& a) {
  return a.quantized && a.q_dtype == SPATTEN_BF16 && (a.d_h == 64 || a.d_h == 128) && a.n_q > 1;
}

int32_t attn_tc_launch(const AttnProblem& p, cudaStream_t st) {
  if (p.a.d_h == 64) return launch<64>(p, st);
  return launch<128>(p, st);
}

}  // namespace spt
