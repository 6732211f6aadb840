// K2: prefill attention with importance on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// SpAtten §II "Attention mechanism" (S = Q K^T scaled, row softmax, P V), §II "Cascade pruning"
// (token importance = column sums of P; head importance = sum |O|), §IV.E "Progressive
// Quantization" (MSB pass; rows whose max probability is below the threshold are recomputed with
// the LSBs).  One CTA = (sequence, kept head, 128 query rows); thread i owns query row i, which
// is TMEM lane i of every accumulator.
//
// Exactness of the operands: K and V are stored as 12-bit codes q = 16*MSB + LSB; 16*MSB
// (|.| <= 2048, 8 significant bits) and LSB (0..15) are both exact in bf16, so the MMAs see the
// codes without rounding and the scale s is applied to the float32 accumulators:
//   S_msb = s_k * sm * (Q . (16 MSB)^T),   S_full = S_msb + s_k * sm * (Q . LSB^T)
//   O     = s_v * (P . 16 MSB_v  [+ P . LSB_v for refetched rows])
// The LSB products go to their own TMEM columns; each softmax thread adds them only for its own
// row when that row is refetched, so no masked operand copies are needed.
//
// Shared-memory operands use the UMMA 128-byte-swizzle layouts: Q, K and P K-major; V MN-major,
// which is simply key rows of d_h bf16 values (the same bytes the K tile layout would hold).
// TMEM (512 columns): S [0,128), C = Q.LSB^T [128,256), O [256, 256+d_h), O_lsb after it.
//
// Passes over the keys, in 128-key tiles (MSB codes dequantized to bf16 in shared memory):
//   A   S_msb -> online row max / exp-sum (base-2 exponentials on MUFU) -> flag = 1/ell < theta
//   A'  only if a row of the tile is flagged: S and C -> statistics of the flagged rows
//   B   S (+C) -> P = exp(S - m)/ell (float32) -> column sums by a 31-shuffle butterfly per 32
//       keys (deterministic) -> P in bf16 to shared memory -> O += P V16 (+ O_lsb += P V_lsb)
// Column sums go to the per-CTA partial buffer; attn_reduce adds them in a fixed order.
// Every mbarrier wait is bounded: on timeout the CTA reports SPATTEN_E_TIMEOUT, frees its TMEM
// and returns.
#include "attention.cuh"
#include "tc_ptx.cuh"

namespace spt {
namespace {

using namespace tc;

constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 24;   // polls of a single mbarrier phase before giving up
constexpr float kLog2e = 1.4426950408889634f;

template <int DH>
struct Layout {
  static constexpr uint32_t kTile = 128u * DH * 2u;        // 128 rows x d_h bf16
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;
  static constexpr uint32_t kKL = kK + kTile;
  static constexpr uint32_t kV = kKL + kTile;
  static constexpr uint32_t kVL = kV + kTile;
  static constexpr uint32_t kP = kVL + kTile;
  static constexpr uint32_t kEnd = kP + 128u * 128u * 2u;
  // at least 116 KB so that one CTA (and its 512 TMEM columns) owns an SM
  static constexpr uint32_t kSmem = (kEnd + 1024u) < 118784u ? 118784u : (kEnd + 1024u);
};

// byte offset of 16-byte chunk c8 (8 consecutive bf16 of a row) in a [128 rows x W] tile stored
// as W/64 column blocks of 128 rows x 128 bytes, 128-byte swizzled
__device__ __forceinline__ uint32_t tile_off(uint32_t row, uint32_t c8) {
  return (c8 >> 3) * 16384u + sw128_offset(row, c8 & 7u);
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

template <int DH>
struct Ctx {
  const spatten_attn_args* a;
  uint8_t* smem;
  int b, h, t0;
  int64_t plane0;          // (b*H + h) * kv_cap
  const int32_t* kv_idx;   // row list of this sequence or nullptr
};

// dequantize keys [t*128, t*128+128) of a K or V plane (MSB -> 16*MSB, LSB -> LSB) into a tile
template <int DH>
__device__ __forceinline__ void load_codes(const Ctx<DH>& c, int t, const int8_t* msb, const uint8_t* lsb,
                                           uint32_t off_hi, uint32_t off_lo) {
  const spatten_attn_args& a = *c.a;
  constexpr int L16 = DH / 16;
  for (int e = threadIdx.x; e < 128 * L16; e += kThreads) {
    const int r = e / L16, c16 = e % L16;
    const int key = t * 128 + r;
    uint32_t hi[8], lo[8];
    if (key < a.n_kv) {
      const int64_t row = c.plane0 + (c.kv_idx ? c.kv_idx[key] : key);
      cvt16_s8x16(__ldg(reinterpret_cast<const uint4*>(msb + row * DH) + c16), hi);
      if (lsb) cvt_u4x16(__ldg(reinterpret_cast<const uint2*>(lsb + row * (DH / 2)) + c16), lo);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) hi[i] = lo[i] = 0u;
    }
    uint4* d0 = reinterpret_cast<uint4*>(c.smem + off_hi + tile_off(r, 2 * c16));
    uint4* d1 = reinterpret_cast<uint4*>(c.smem + off_hi + tile_off(r, 2 * c16 + 1));
    *d0 = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *d1 = make_uint4(hi[4], hi[5], hi[6], hi[7]);
    if (lsb) {
      *reinterpret_cast<uint4*>(c.smem + off_lo + tile_off(r, 2 * c16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(c.smem + off_lo + tile_off(r, 2 * c16 + 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
    }
  }
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

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(AttnProblem p) {
  using LY = Layout<DH>;
  const spatten_attn_args& a = p.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ float colred[4][128];
  __shared__ float hred[4];

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
        *reinterpret_cast<uint4*>(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok + static_cast<int64_t>(h) * DH + c8 * 8) =
            make_uint4(0, 0, 0, 0);
    }
    return;
  }

  if (warp == 0) {
    tmem_alloc(&tmem_base_s, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tmem_base_s;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem, tC = tmem + 128, tO = tmem + 256, tO2 = tmem + 256 + DH;
  uint32_t phase = 0;
  bool aborted = false;

  Ctx<DH> c{&a, smem, b, h, i0, (static_cast<int64_t>(b) * a.H + h) * a.kv_cap,
            a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr};

  // ---- Q tile ---------------------------------------------------------------------------------
  {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
    for (int e = tid; e < 128 * (DH / 8); e += kThreads) {
      const int r = e / (DH / 8), c8 = e % (DH / 8), i = i0 + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (i < a.n_q)
        v = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * a.n_q + i) * a.q_ld_tok +
                                                 static_cast<int64_t>(h) * DH) + c8);
      *reinterpret_cast<uint4*>(smem + LY::kQ + tile_off(r, c8)) = v;
    }
  }

  const uint32_t sQ = smem_u32(smem + LY::kQ), sK = smem_u32(smem + LY::kK), sKL = smem_u32(smem + LY::kKL);
  const uint32_t sV = smem_u32(smem + LY::kV), sVL = smem_u32(smem + LY::kVL), sP = smem_u32(smem + LY::kP);
  constexpr uint32_t kIdQK = idesc_bf16(128, 128, false, false);
  constexpr uint32_t kIdPV = idesc_bf16(128, DH, false, true);

  // S (and C) for the key tile in shared memory; called by every thread, issued by thread 0
  auto issue_qk = [&](bool with_lsb) {
    if (tid == 0) {
      tc_after_sync();
#pragma unroll
      for (int s = 0; s < DH / 16; ++s) {
        const uint32_t koff = (s >> 2) * 16384u + (s & 3) * 32u;
        mma_bf16(tS, desc_sw128(sQ + koff, 16, 1024), desc_sw128(sK + koff, 16, 1024), kIdQK, s > 0);
      }
      if (with_lsb) {
#pragma unroll
        for (int s = 0; s < DH / 16; ++s) {
          const uint32_t koff = (s >> 2) * 16384u + (s & 3) * 32u;
          mma_bf16(tC, desc_sw128(sQ + koff, 16, 1024), desc_sw128(sKL + koff, 16, 1024), kIdQK, s > 0);
        }
      }
      mma_commit(&bar);
    }
  };
  auto issue_pv = [&](bool with_lsb, bool accumulate) {
    if (tid == 0) {
      tc_after_sync();
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t poff = (s >> 2) * 16384u + (s & 3) * 32u;
        const uint32_t voff = s * 2048u;
        mma_bf16(tO, desc_sw128(sP + poff, 16, 1024), desc_sw128(sV + voff, 16384, 1024), kIdPV, accumulate || s > 0);
        if (with_lsb)
          mma_bf16(tO2, desc_sw128(sP + poff, 16, 1024), desc_sw128(sVL + voff, 16384, 1024), kIdPV,
                   accumulate || s > 0);
      }
      mma_commit(&bar);
    }
  };
  auto wait_mma = [&]() {
    const bool ok = mbar_wait(&bar, phase, kWaitLimit);
    phase ^= 1u;
    tc_after_sync();
    if (__syncthreads_or(!ok)) aborted = true;
  };

  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const float c2 = a.k_scale[bh] * a.sm_scale * kLog2e;   // raw accumulator -> log2-domain score
  const int row = tid, i = i0 + row;
  const bool row_ok = i < a.n_q;
  const int n_tiles = (a.n_kv + 127) / 128;

  // ---- pass A: MSB statistics --------------------------------------------------------------------
  float m2 = -INFINITY, l = 0.0f;
  for (int t = 0; t < n_tiles && !aborted; ++t) {
    load_codes<DH>(c, t, a.k_msb, nullptr, LY::kK, 0);
    fence_async_smem();
    __syncthreads();
    issue_qk(false);
    wait_mma();
    if (aborted) break;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      float v[32];
      __syncwarp();
      tmem_ld32(tS + lane_base + ch * 32, v);
      tmem_ld_wait();
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        v[j] = (t * 128 + ch * 32 + j < a.n_kv) ? v[j] * c2 : -INFINITY;
        mx = fmaxf(mx, v[j]);
      }
      if (mx == -INFINITY) continue;
      const float mn = fmaxf(m2, mx);
      float add = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) add += ex2(v[j] - mn);
      l = l * ex2(m2 - mn) + add;
      m2 = mn;
    }
    tc_before_sync();
    __syncthreads();
  }
  const bool flag = !aborted && a.quantized && row_ok && (1.0f / l < a.refetch_threshold);
  const bool any_flag = __syncthreads_or(flag) != 0;

  // ---- pass A': full-precision statistics of the flagged rows --------------------------------
  if (any_flag && !aborted) {
    float mf = -INFINITY, lf = 0.0f;
    for (int t = 0; t < n_tiles && !aborted; ++t) {
      load_codes<DH>(c, t, a.k_msb, a.k_lsb, LY::kK, LY::kKL);
      fence_async_smem();
      __syncthreads();
      issue_qk(true);
      wait_mma();
      if (aborted) break;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        float v[32], w[32];
        __syncwarp();
        tmem_ld32(tS + lane_base + ch * 32, v);
        tmem_ld32(tC + lane_base + ch * 32, w);
        tmem_ld_wait();
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = (t * 128 + ch * 32 + j < a.n_kv) ? (v[j] + w[j]) * c2 : -INFINITY;
          mx = fmaxf(mx, v[j]);
        }
        if (mx == -INFINITY) continue;
        const float mn = fmaxf(mf, mx);
        float add = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) add += ex2(v[j] - mn);
        lf = lf * ex2(mf - mn) + add;
        mf = mn;
      }
      tc_before_sync();
      __syncthreads();
    }
    if (flag) {
      m2 = mf;
      l = lf;
    }
  }

  // ---- pass B: probabilities, importance, outputs -------------------------------------------------
  const float inv_l = 1.0f / l;
  const int64_t part_row = ((static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt) * a.n_kv;
  for (int t = 0; t < n_tiles && !aborted; ++t) {
    load_codes<DH>(c, t, a.k_msb, any_flag ? a.k_lsb : nullptr, LY::kK, LY::kKL);
    load_codes<DH>(c, t, a.v_msb, any_flag ? a.v_lsb : nullptr, LY::kV, LY::kVL);
    fence_async_smem();
    __syncthreads();
    issue_qk(any_flag);
    wait_mma();
    if (aborted) break;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      float v[32];
      __syncwarp();
      tmem_ld32(tS + lane_base + ch * 32, v);
      if (any_flag) {
        float w[32];
        tmem_ld32(tC + lane_base + ch * 32, w);
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
        const bool ok = row_ok && (t * 128 + ch * 32 + j < a.n_kv);
        v[j] = ok ? ex2(v[j] * c2 - m2) * inv_l : 0.0f;
      }
      // P row chunk (bf16) into the K-major P tile: columns ch*32 .. ch*32+31
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint32_t c8 = ch * 4 + q4;
        *reinterpret_cast<uint4*>(smem + LY::kP + tile_off(row, c8)) =
            make_uint4(pack_bf16x2(v[8 * q4 + 0], v[8 * q4 + 1]), pack_bf16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                       pack_bf16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_bf16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
      }
      colred[warp][ch * 32 + lane] = warp_colsum32(v);
    }
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    issue_pv(any_flag, t > 0);
    {
      const int key = t * 128 + tid;
      if (key < a.n_kv) p.tok_part[part_row + key] = ((colred[0][tid] + colred[1][tid]) + colred[2][tid]) + colred[3][tid];
    }
    wait_mma();
  }

  // ---- epilogue: O, head importance, flags --------------------------------------------------------
  float habs = 0.0f;
  if (!aborted) {
    const float vs = a.v_scale[bh];
#pragma unroll 1
    for (int ch = 0; ch < DH / 32; ++ch) {
      float v[32];
      __syncwarp();
      tmem_ld32(tO + lane_base + ch * 32, v);
      if (any_flag) {
        float w[32];
        tmem_ld32(tO2 + lane_base + ch * 32, w);
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
  habs = warp_sum(habs);
  const int nflag = __syncthreads_count(flag);
  if (lane == 0) hred[warp] = habs;
  tc_before_sync();
  __syncthreads();
  if (tid == 0) {
    p.head_part[(static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt] = ((hred[0] + hred[1]) + hred[2]) + hred[3];
    if (nflag && a.refetch_count) atomicAdd(a.refetch_count, nflag);
    if (aborted) report(a.dev_status, SPATTEN_E_TIMEOUT);
  }
  if (warp == 0) {
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
                                  static_cast<int>(Layout<DH>::kSmem)));
    configured[dev] = true;
  }
  const int slots = p.a.H_kept + (p.a.zero_pruned_heads ? p.a.H - p.a.H_kept : 0);
  attn_tc_kernel<DH><<<dim3(p.n_qt, slots, p.a.B), kThreads, Layout<DH>::kSmem, st>>>(p);
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
