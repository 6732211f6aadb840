// K2: prefill attention with importance on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// SpAtten §II "Attention mechanism" (S = Q K^T scaled, row softmax, P V), §II "Cascade pruning"
// (token importance = column sums of P; head importance = sum |O|), §IV.E "Progressive
// Quantization" (MSB pass; rows whose max probability is below the threshold are recomputed with
// the LSBs).
//
// Exact operands: K and V are 12-bit codes q = 16*MSB + LSB; 16*MSB (in [-2048, 2032]) and LSB
// (0..15) are exact in fp16, so the MMAs (kind::f16 with fp16 A and B, f32 accumulate) see the
// codes unrounded and the scales multiply the float32 accumulators:
//   S = s_k*sm*(Q.(16 MSB)^T [+ Q.LSB^T]),  O = s_v*(P.16 MSB_v [+ P.LSB_v]).
// The bf16 query tile is converted to fp16 on its way to shared memory (exact for magnitudes in
// [2^-14, 65504]; smaller ones keep fp16 subnormal precision, larger ones saturate) and P is
// stored as fp16 (11 significant bits).
//
// Two kernels per layer:
//  MAIN  persistent: one CTA per SM walks the work items (sequence, kept head, 256 query rows) with
//        a stride of the grid; TMEM, barriers and all ring counters live across items, so the
//        producers load the next item's query tile and first key tiles, and the MMA warp issues its
//        first score MMAs, while the softmax warps finish the current item.  d_h 64: 512 threads:
//          warps 0-7   two softmax warpgroups; warpgroup g owns query rows 128g..128g+127 of the
//                      CTA, thread r of a warpgroup is TMEM lane r of that warpgroup's S and O
//          warps 8-14  producers: the item's query tile, then K/V MSB tiles converted into
//                      2-stage rings
//          warp 15     MMA issue (lane 0) and TMEM allocation
//        The softmax warpgroups run with more registers than the launch gives (setmaxnreg),
//        warpgroups 2-3 with fewer.  d_h 128: 384 threads, producer warps 8-10, MMA warp 11.
//        pass A computes S_msb tile by tile (the two warpgroups' tiles alternate on the tensor
//        core while the other warpgroup runs its softmax) -> row max / exp-sum -> refetch flags;
//        the flagged rows of the CTA are written, ascending, to a packed list.  Pass B computes
//        P = exp(S - m)/ell for the other rows (float32), column sums by a 31-shuffle butterfly
//        (deterministic), P in fp16 to shared memory, O += P V.  Flagged rows contribute nothing
//        here.
//  FULL  one CTA = 128 consecutive entries of the head's flagged rows (the MAIN lists of its pair
//        tiles concatenated in order; launched only when theta > 0; CTAs past the end exit at
//        once), 256 threads (4 softmax, 3 producer, 1 MMA warps): the same two passes with
//        S = Q.(16 MSB)^T + Q.LSB^T and O = P.16 MSB_v + P.LSB_v accumulated in the same TMEM
//        columns, reading the LSB planes only for heads with flagged rows.
// Producers: without an index list the raw code rows of a key tile are contiguous, so one thread
// keeps several tiles in flight with 1-D bulk copies (TMA engine) into a staging ring, and the
// producer warps convert staged int8 / packed-nibble tiles to swizzled fp16 shared -> shared (a
// byte placed under the fp16 exponent byte 0x64 reads as 1024 + byte; one fp16 FMA or add per pair
// of codes removes the offset, no int-to-float conversions).
// Partial column sums (per 128-row tile) and sum |O| go to the workspace; attn_reduce adds them in
// a fixed order, so reruns are bit-identical.
// Operand layouts: UMMA 128-byte swizzle; Q, K, P K-major; V MN-major (plain key rows).  Key tiles
// hold 16 KB of fp16 codes: 128 keys at d_h = 64, 64 keys at d_h = 128.  Every mbarrier wait is
// bounded: on timeout the CTA reports SPATTEN_E_TIMEOUT, frees its TMEM and returns.
#include <cuda_fp16.h>

#include "attention.cuh"
#include "exp2_poly.cuh"
#include "tc_ptx.cuh"

namespace spt {
namespace {

using namespace tc;

constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kProducerThreads = 96;    // refetch kernel: warps 4-6
// main kernel, d_h 64: 16 warps = softmax warpgroups 0 and 1, producer warps 8-14, MMA warp 15.
// The two softmax warpgroups raise their register limit and the other two lower theirs
// (setmaxnreg), so that seven producer warps fit beside softmax threads that need 160 registers:
// 256 x 168 + 256 x 88 = 65536 = 512 threads x 128 registers at launch.  d_h 128: 12 warps,
// producer warps 8-10, MMA warp 11, no split (168 registers per thread at launch).
template <int DH> constexpr int kMainThreads = DH == 64 ? 512 : 384;
template <int DH> constexpr int kMainProducers = kMainThreads<DH> - 256 - 32;
template <int DH> constexpr int kMainMmaWarp = kMainThreads<DH> / 32 - 1;
constexpr uint32_t kSoftmaxRegs = 168, kOtherRegs = 88;
static_assert(256 * kSoftmaxRegs + 256 * kOtherRegs <= 65536, "register split");
// Of every four pairs of softmax exponentials in the main kernel, this many are computed by the
// FMA-pipe polynomial (exp2_poly2) and the rest by the ex2 instruction: the two units then share
// the work.
#ifndef SPT_EXP2_POLY_PAIRS
#define SPT_EXP2_POLY_PAIRS 1
#endif
constexpr int kPolyPairs = SPT_EXP2_POLY_PAIRS;   // BERT step: 0 pairs -0.2 %, 2 pairs -3 % against 1

// byte offset of 16-byte chunk c8 of `row` in a tile whose 64-element column blocks each hold
// `rows` rows of 128 bytes (128-byte swizzle)
__device__ __forceinline__ uint32_t tile_off(uint32_t row, uint32_t c8, uint32_t rows) {
  return (c8 >> 3) * rows * 128u + sw128_offset(row, c8 & 7u);
}

// Code tiles enter the tensor cores as fp16, in which every code value is exact (16 MSB lies in
// [-2048, 2032], LSB in [0, 15]).  Conversion without int-to-float instructions: a code byte u
// placed under the high byte 0x64 is the fp16 number 1024 + u.
// sixteen signed MSB codes -> eight fp16 pairs of 16 * MSB: the biased byte u = MSB + 128 gives
// 1024 + u, and 16 (1024 + u) - 18432 = 16 MSB is exact in one fp16 FMA
__device__ __forceinline__ void cvt16_s8x16(uint4 raw, uint32_t* out8) {
  const uint32_t w[4] = {raw.x ^ 0x80808080u, raw.y ^ 0x80808080u, raw.z ^ 0x80808080u, raw.w ^ 0x80808080u};
  const __half2 mul = __halves2half2(__float2half_rn(16.0f), __float2half_rn(16.0f));
  const __half2 add = __halves2half2(__float2half_rn(-18432.0f), __float2half_rn(-18432.0f));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t p0 = __byte_perm(w[i], 0x64646464u, 0x5140u), p1 = __byte_perm(w[i], 0x64646464u, 0x5342u);
    __half2 h0 = __hfma2(*reinterpret_cast<__half2*>(&p0), mul, add);
    __half2 h1 = __hfma2(*reinterpret_cast<__half2*>(&p1), mul, add);
    out8[2 * i] = *reinterpret_cast<uint32_t*>(&h0);
    out8[2 * i + 1] = *reinterpret_cast<uint32_t*>(&h1);
  }
}
// sixteen packed LSB codes (element 2k in bits 8k..8k+3, 2k+1 in bits 8k+4..8k+7 of a word) ->
// eight fp16 pairs
__device__ __forceinline__ void cvt_u4x16(uint2 raw, uint32_t* out8) {
  const uint32_t w[2] = {raw.x, raw.y};
  const __half2 off = __halves2half2(__float2half_rn(-1024.0f), __float2half_rn(-1024.0f));
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t p = (__byte_perm(lo, hi, static_cast<uint32_t>(k | ((4 + k) << 8))) & 0x00FF00FFu) | 0x64006400u;
      __half2 h = __hadd2(*reinterpret_cast<__half2*>(&p), off);
      out8[4 * i + k] = *reinterpret_cast<uint32_t*>(&h);
    }
  }
}
// Range check of bf16 values against fp16: the running maximum `mx` of the sign-cleared bit
// patterns (two 16-bit maxima per word; patterns order like magnitudes, NaNs above infinity) is
// out of range from 0x4780 up: magnitude 65536 or more (bf16 has no value in (65504, 65536)),
// infinity or NaN.
__device__ __forceinline__ uint32_t bf16x8_absmax(uint4 u, uint32_t mx) {
  constexpr uint32_t M = 0x7FFF7FFFu;
  return __vmaxu2(mx, __vmaxu2(__vmaxu2(u.x & M, u.y & M), __vmaxu2(u.z & M, u.w & M)));
}
__device__ __forceinline__ bool bf16_absmax_out_of_f16(uint32_t mx) {
  return (mx & 0xFFFFu) >= 0x4780u || (mx >> 16) >= 0x4780u;
}
// eight bf16 values -> four fp16 pairs (the query tile); exact for magnitudes in [2^-14, 65504]
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = pack_f16x2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// 16-byte asynchronous global -> shared copy (no register staging); src_bytes 0 zero-fills
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// bounded wait that also gives up once another role has aborted; `limit` polls of one phase
// before giving up (AttnProblem::wait_limit)
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

// after an abort: wait, with a bound of its own, for a phase that work already in flight (a bulk
// copy, committed MMAs) will complete, so shared memory and TMEM are not released under it
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 22); ++i)
    if (mbar_try_wait(bar, parity)) return;
}

// The AND of `ok` over the 128 threads of a softmax warpgroup (named barrier `id`): after a wait,
// every thread of the group takes the same branch, so no thread can leave a group barrier or a
// warp-collective TMEM load short of participants after a timeout.
__device__ __forceinline__ bool wg_all(bool ok, int id) {
  uint32_t r;
  asm volatile(
      "{\n"
      ".reg .pred p, q;\n"
      "setp.ne.u32 p, %1, 0;\n"
      "bar.red.and.pred q, %2, 128, p;\n"
      "selp.u32 %0, 1, 0, q;\n"
      "}\n"
      : "=r"(r)
      : "r"(ok ? 1u : 0u), "r"(id)
      : "memory");
  return r != 0;
}

// paired float32 arithmetic (two lanes per instruction on sm_100)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// 2^x of a pair: pair `q` of each group of four takes the FMA-pipe polynomial when q < kPolyPairs,
// else the ex2 instruction (q is a compile-time index, so the choice costs nothing)
template <int Q>
__device__ __forceinline__ float2 exp2_pair(float2 x) {
  if constexpr ((Q & 3) < kPolyPairs) return exp2_poly2(x);
  else return make_float2(ex2(x.x), ex2(x.y));
}

// column sums over the 32 rows of a warp for two 32-column arrays: afterwards lane l holds the
// sums of column l of each (two independent butterfly chains, twice the ILP)
__device__ __forceinline__ void warp_colsum32x2(float* v, float* w, float& sv, float& sw) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send_v = upper ? v[j] : v[j + off];
      const float keep_v = upper ? v[j + off] : v[j];
      const float send_w = upper ? w[j] : w[j + off];
      const float keep_w = upper ? w[j + off] : w[j];
      v[j] = keep_v + __shfl_xor_sync(0xffffffffu, send_v, off);
      w[j] = keep_w + __shfl_xor_sync(0xffffffffu, send_w, off);
    }
  }
  sv = v[0];
  sw = w[0];
}

// the same update over 64 raw scores of a full chunk: c2 (> 0) carries the softmax scale into the
// log2 domain, max(c2 v) = c2 max(v), and each exponent is one fused c2 v - m
__device__ __forceinline__ void stats64_scaled(const float* v, float c2, float& m2, float& l) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    mx[k] = v[k];
#pragma unroll
    for (int j = 1; j < 8; ++j) mx[k] = fmaxf(mx[k], v[k + 8 * j]);
  }
  const float mm = c2 * fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
  const float mn = fmaxf(m2, mm);
  const float2 c2x2 = make_float2(c2, c2), nmn = make_float2(-mn, -mn);
  float2 s0 = make_float2(0.0f, 0.0f), s1 = s0;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    s0 = fadd2(s0, exp2_pair<0>(ffma2(make_float2(v[2 * j + 0], v[2 * j + 1]), c2x2, nmn)));
    s1 = fadd2(s1, exp2_pair<1>(ffma2(make_float2(v[2 * j + 2], v[2 * j + 3]), c2x2, nmn)));
    s0 = fadd2(s0, exp2_pair<2>(ffma2(make_float2(v[2 * j + 4], v[2 * j + 5]), c2x2, nmn)));
    s1 = fadd2(s1, exp2_pair<3>(ffma2(make_float2(v[2 * j + 6], v[2 * j + 7]), c2x2, nmn)));
  }
  l = l * ex2(m2 - mn) + ((s0.x + s1.x) + (s0.y + s1.y));
  m2 = mn;
}

// running max / exp-sum update over 64 log2-domain scores (independent partial sums)
__device__ __forceinline__ void stats64(const float* v, float& m2, float& l) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    mx[k] = v[k];
#pragma unroll
    for (int j = 1; j < 8; ++j) mx[k] = fmaxf(mx[k], v[k + 8 * j]);
  }
  const float mm = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
  if (mm == -INFINITY) return;
  const float mn = fmaxf(m2, mm);
  float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int j = 0; j < 64; ++j) s[j & 3] += ex2(v[j] - mn);
  l = l * ex2(m2 - mn) + ((s[0] + s[1]) + (s[2] + s[3]));
  m2 = mn;
}

// 16·MSB + LSB, pair by pair: the 12-bit code itself, an integer of magnitude at most 2048, so the
// fp16 sum is exact and one MMA over the combined tile replaces an MSB and an LSB product
__device__ __forceinline__ void add_f16x8(uint32_t* hi, const uint32_t* lo) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const __half2 s = __hadd2(*reinterpret_cast<const __half2*>(&hi[q]), *reinterpret_cast<const __half2*>(&lo[q]));
    hi[q] = *reinterpret_cast<const uint32_t*>(&s);
  }
}

template <int DH, int KT, int NP>
__device__ __forceinline__ void produce_tile(uint8_t* smem, int t, int n_kv, int64_t plane0, const int32_t* kv_idx,
                                             const int8_t* msb, const uint8_t* lsb, uint32_t off_hi, int ptid,
                                             const uint8_t* keep) {
  constexpr int L16 = DH / 16;
  for (int e = ptid; e < KT * L16; e += NP) {
    const int r = e / L16, c16 = e % L16;
    const int key = t * KT + r;
    uint32_t hi[8], lo[8];
    if (key < n_kv && (!keep || keep[key])) {
      const int64_t prow = plane0 + (kv_idx ? kv_idx[key] : key);
      cvt16_s8x16(__ldg(reinterpret_cast<const uint4*>(msb + prow * DH) + c16), hi);
      if (lsb) {
        cvt_u4x16(__ldg(reinterpret_cast<const uint2*>(lsb + prow * (DH / 2)) + c16), lo);
        add_f16x8(hi, lo);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) hi[q] = 0u;
    }
    *reinterpret_cast<uint4*>(smem + off_hi + tile_off(r, 2 * c16, KT)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + off_hi + tile_off(r, 2 * c16 + 1, KT)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
  }
  fence_async_smem();
}

// same conversion from a staged raw tile in shared memory: MSB rows (DH bytes each) at raw,
// packed LSB rows (DH/2 bytes) at raw + KT*DH; rows >= valid are zero-filled
// keep (V tiles under local value pruning): row r of the tile is kept iff keep[r] != 0; dropped
// rows are zero-filled like the rows past the end
template <int DH, int KT, bool KEEP, int NP>
__device__ __forceinline__ void convert_staged(uint8_t* smem, const uint8_t* raw, bool with_lsb, int valid,
                                               uint32_t off_hi, int ptid, const uint8_t* keep) {
  constexpr int L16 = DH / 16;
  constexpr int TOTAL = KT * L16;
  constexpr int NIT = (TOTAL + NP - 1) / NP;
  // every staged read of this thread first (all in flight together), then the conversions
  uint4 m[NIT];
  uint2 lb[NIT];
#pragma unroll
  for (int i = 0; i < NIT; ++i) {
    const int e = ptid + i * NP;
    const int r = e / L16, c16 = e % L16;
    m[i] = make_uint4(0u, 0u, 0u, 0u);
    lb[i] = make_uint2(0u, 0u);
    if (e < TOTAL && r < valid && (!KEEP || keep[r])) {
      m[i] = *reinterpret_cast<const uint4*>(raw + r * DH + c16 * 16);
      if (with_lsb) lb[i] = *reinterpret_cast<const uint2*>(raw + KT * DH + r * (DH / 2) + c16 * 8);
    }
  }
#pragma unroll
  for (int i = 0; i < NIT; ++i) {
    const int e = ptid + i * NP;
    if (e >= TOTAL) break;
    const int r = e / L16, c16 = e % L16;
    uint32_t hi[8], lo[8];
    if (r < valid && (!KEEP || keep[r])) {
      cvt16_s8x16(m[i], hi);
      if (with_lsb) {
        cvt_u4x16(lb[i], lo);
        add_f16x8(hi, lo);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) hi[q] = 0u;
    }
    *reinterpret_cast<uint4*>(smem + off_hi + tile_off(r, 2 * c16, KT)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + off_hi + tile_off(r, 2 * c16 + 1, KT)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
  }
  fence_async_smem();
}

// The producers' work as one job stream: jobs 0..T-1 are the K tiles of pass A, then pass B
// alternates K(t), V(t).  Without an index list the raw code rows of a tile are contiguous, so one
// loader thread keeps RS tiles in flight with 1-D bulk copies (TMA engine) into a staging ring and
// all producer threads convert staged tiles shared -> shared; with an index list they load rows
// directly.  `emit(is_v, t, stage_dst_hi, stage_dst_lo)` gives the destination of the converted
// tile and performs the ring handshake around `fill`.
template <int DH, int KT, int RS, int NP>   // NP producer threads
struct JobStream {
  static constexpr uint32_t kMsb = KT * DH;
  uint8_t* smem;
  uint32_t o_raw, raw_bytes;   // staging ring: RS slots of raw_bytes
  uint64_t* raw_full;          // [RS]
  uint64_t* raw_empty;         // [RS], count NP
  const spatten_attn_args* a;
  int64_t plane0;
  int n_tiles;
  bool with_lsb;
  int ptid;
  volatile int* abort_flag;
  uint32_t g0 = 0;       // global index of this stream's job 0 in the staging ring's sequence
  uint32_t issued = 0;   // jobs of this stream issued so far (loader)
  uint32_t consumed = 0; // jobs of this stream converted so far
  const uint8_t* vmask = nullptr;   // [n_kv] V vectors kept (local value pruning) or NULL
  uint32_t wlim = kDefaultWaitLimit;  // polls of one wait before giving up

  __device__ __forceinline__ int jobs() const { return 3 * n_tiles; }
  __device__ __forceinline__ void job(int j, bool& is_v, int& t) const {
    if (j < n_tiles) {
      is_v = false;
      t = j;
    } else {
      is_v = ((j - n_tiles) & 1) != 0;
      t = (j - n_tiles) >> 1;
    }
  }
  __device__ __forceinline__ int valid_rows(int t) const { return min(KT, a->n_kv - t * KT); }
  // loader only: issue jobs up to j + RS - 1
  __device__ __forceinline__ bool issue_ahead(int j) {
    while (static_cast<int>(issued) < jobs() && static_cast<int>(issued) < j + RS) {
      const uint32_t jn = issued;
      const uint32_t gj = g0 + jn;
      const uint32_t st = gj % RS;
      if (!wait_bar(&raw_empty[st], ((gj / RS) & 1u) ^ 1u, abort_flag, wlim)) return false;
      bool is_v;
      int t;
      job(static_cast<int>(jn), is_v, t);
      const int rows = valid_rows(t);
      const int64_t row0 = plane0 + static_cast<int64_t>(t) * KT;
      const uint32_t mb = static_cast<uint32_t>(rows) * DH, lb = with_lsb ? mb / 2 : 0u;
      uint8_t* dst = smem + o_raw + st * raw_bytes;
      mbar_arrive_expect_tx(&raw_full[st], mb + lb);
      bulk_g2s(dst, (is_v ? a->v_msb : a->k_msb) + row0 * DH, mb, &raw_full[st]);
      if (with_lsb) bulk_g2s(dst + kMsb, (is_v ? a->v_lsb : a->k_lsb) + row0 * (DH / 2), lb, &raw_full[st]);
      ++issued;
    }
    return true;
  }
  // convert job j into the fp16 tile at off_hi (16·MSB, or with the LSB plane the combined
  // 16·MSB + LSB); returns false on abort
  __device__ __forceinline__ bool convert(int j, uint32_t off_hi, const int32_t* kv_idx) {
    bool is_v;
    int t;
    job(j, is_v, t);
    const uint8_t* keep = (is_v && vmask) ? vmask : nullptr;
    if (kv_idx) {
      produce_tile<DH, KT, NP>(smem, t, a->n_kv, plane0, kv_idx, is_v ? a->v_msb : a->k_msb,
                           with_lsb ? (is_v ? a->v_lsb : a->k_lsb) : nullptr, off_hi, ptid, keep);
      return true;
    }
    const uint32_t gj = g0 + static_cast<uint32_t>(j);
    const uint32_t st = gj % RS;
    if (!wait_bar(&raw_full[st], (gj / RS) & 1u, abort_flag, wlim)) return false;
    if (keep)
      convert_staged<DH, KT, true, NP>(smem, smem + o_raw + st * raw_bytes, with_lsb, valid_rows(t), off_hi, ptid,
                                   keep + t * KT);
    else
      convert_staged<DH, KT, false, NP>(smem, smem + o_raw + st * raw_bytes, with_lsb, valid_rows(t), off_hi, ptid,
                                    nullptr);
    mbar_arrive(&raw_empty[st]);
    ++consumed;
    return true;
  }
};

// QK^T into `d` (accumulate onto it when acc != 0), A = Q tile [128 x DH], B = key tile [KT x DH]
template <int DH, int KT>
__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t sQ, uint32_t sK, uint32_t acc) {
  constexpr uint32_t id = idesc_f16(128, KT, false, false);
#pragma unroll
  for (int s = 0; s < DH / 16; ++s) {
    const uint32_t qoff = (s >> 2) * 16384u + (s & 3) * 32u;
    const uint32_t koff = (s >> 2) * (KT * 128u) + (s & 3) * 32u;
    mma_f16(d, desc_sw128(sQ + qoff, 16, 1024), desc_sw128(sK + koff, 16, 1024), id, (acc || s > 0) ? 1u : 0u);
  }
}
// P V into `d`: A = P tile [128 x KT] K-major, B = V tile [KT keys x DH] MN-major
template <int DH, int KT>
__device__ __forceinline__ void mma_pv(uint32_t d, uint32_t sP, uint32_t sV, uint32_t acc) {
  constexpr uint32_t id = idesc_f16(128, DH, false, true);
#pragma unroll
  for (int s = 0; s < KT / 16; ++s) {
    const uint32_t poff = (s >> 2) * 16384u + (s & 3) * 32u;
    mma_f16(d, desc_sw128(sP + poff, 16, 1024), desc_sw128(sV + s * 2048u, KT * 128u, 1024), id,
             (acc || s > 0) ? 1u : 0u);
  }
}

// S^T = K Q^T into `d`: A = key tile [KT keys x DH] (K-major), B = one warpgroup's query tile
// [128 rows x DH] (K-major).  TMEM lane = key, column = query row.
template <int DH, int KT>
__device__ __forceinline__ void mma_kq(uint32_t d, uint32_t sK, uint32_t sQ) {
  constexpr uint32_t id = idesc_f16(KT, 128, false, false);
#pragma unroll
  for (int s = 0; s < DH / 16; ++s) {
    const uint32_t koff = (s >> 2) * (KT * 128u) + (s & 3) * 32u;
    const uint32_t qoff = (s >> 2) * 16384u + (s & 3) * 32u;
    mma_f16(d, desc_sw128(sK + koff, 16, 1024), desc_sw128(sQ + qoff, 16, 1024), id, s > 0 ? 1u : 0u);
  }
}
// P V into `d` with P stored MN-major (query rows contiguous): A = P tile [128 rows x KT keys] in
// two 64-row blocks KT*128 bytes apart with 8-key groups 1024 bytes apart; B = V tile MN-major
template <int DH, int KT>
__device__ __forceinline__ void mma_pv_mn(uint32_t d, uint32_t sP, uint32_t sV, uint32_t acc) {
  constexpr uint32_t id = idesc_f16(128, DH, true, true);
#pragma unroll
  for (int s = 0; s < KT / 16; ++s)
    mma_f16(d, desc_sw128(sP + s * 2048u, KT * 128u, 1024), desc_sw128(sV + s * 2048u, KT * 128u, 1024), id,
            (acc || s > 0) ? 1u : 0u);
}

__device__ __forceinline__ void store_o_row(__nv_bfloat16* dst, const float* v, float vs, float& habs) {
  uint32_t pk[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float x0 = v[2 * j] * vs, x1 = v[2 * j + 1] * vs;
    habs += fabsf(x0) + fabsf(x1);
    pk[j] = pack_bf16x2(x0, x1);
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) d4[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
}

// =================================================================================================
// MAIN kernel
// =================================================================================================
template <int DH>
struct MainCfg {
  // d_h = 64: the probability pass runs transposed (S^T = K Q^T, one key per TMEM lane, P written
  // MN-major); d_h = 128: row orientation with shuffle column sums (its 128-key tiles would not
  // fit the shared-memory budget)
  static constexpr bool kT = DH == 64;
  static constexpr int KT = DH == 64 ? 128 : 64;
  static constexpr int NST = 2;                  // fp16 K and V ring stages
  // d_h = 64: the next item's query tile is copied into a second buffer while the current item
  // runs (cp.async, converted in place once the current item's key jobs are done); d_h = 128 has
  // no room for a second buffer and loads the query tile between items
  static constexpr int NQ = DH == 64 ? 2 : 1;
  static constexpr int RS = DH == 64 ? 3 : 4;    // raw code tiles in flight (bulk copies; d_h 64: 4 measured 0.3 % slower)
  static constexpr uint32_t QB = 128u * DH * 2u;
  static constexpr uint32_t TB = static_cast<uint32_t>(KT) * DH * 2u;
  static constexpr uint32_t PB = 128u * KT * 2u;
  static constexpr uint32_t RAWB = static_cast<uint32_t>(KT) * DH;   // one raw MSB tile
  static constexpr uint32_t oQ = 0;              // NQ buffers of 2 query tiles (one per warpgroup)
  static constexpr uint32_t oK = NQ * 2 * QB;    // NST stages
  static constexpr uint32_t oV = oK + NST * TB;  // NST stages
  static constexpr uint32_t oP = oV + NST * TB;  // one P tile per warpgroup
  static constexpr uint32_t oRaw = oP + 2 * PB;  // RS staging slots
  static constexpr uint32_t kSmem = oRaw + RS * RAWB + 1024u;
  static constexpr uint32_t tS = 0;              // + g * KT
  static constexpr uint32_t tO = 2u * KT;        // + g * DH
};

enum : int { M_QF = 0, M_QE = 2, M_OE = 4, M_KF = 5, M_KE = 7, M_VF = 9, M_VE = 11, M_SF = 13, M_SR = 15, M_PF = 17,
             M_PE = 19, M_OD = 21, M_RF = 22, M_RE = 26, M_DR = 30, M_N = 31 };   // M_QF, M_QE: one per query buffer

// AND of `ok` over the 256 softmax threads of a CTA (named barrier 3)
__device__ __forceinline__ bool softmax_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n"
      ".reg .pred p, q;\n"
      "setp.ne.u32 p, %1, 0;\n"
      "bar.red.and.pred q, 3, 256, p;\n"
      "selp.u32 %0, 1, 0, q;\n"
      "}\n"
      : "=r"(r)
      : "r"(ok ? 1u : 0u)
      : "memory");
  return r != 0;
}

// Persistent: one CTA per SM walks the work items (sequence, kept head, 256-row pair) with a
// stride of gridDim.x; TMEM, barriers and every ring counter live across items, so the producers
// load the next item's query tile and first key tiles, and the MMA warp issues its first score
// MMAs, while the softmax warps finish the previous item.
// Zero-filled outputs of the pruned heads (slots H_kept .. H-1), shared out over the softmax warps
// of all CTAs before their first scores arrive (the stores overlap the first tiles' loads): warp w
// of the grid takes the units (sequence, pruned slot, 64 query rows) w, w + 8 * gridDim.x, ...
template <int DH>
__device__ __forceinline__ void zero_pruned_share(const spatten_attn_args& a, __nv_bfloat16* o, int warp, int lane) {
  constexpr int kRows = 64, C8 = DH / 8;
  const int np = a.H - a.H_kept;
  const int rblk = (a.n_q + kRows - 1) / kRows;
  const int64_t units = static_cast<int64_t>(a.B) * np * rblk;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * 8 + warp; u < units; u += static_cast<int64_t>(gridDim.x) * 8) {
    const int rb = static_cast<int>(u % rblk);
    const int ps = static_cast<int>((u / rblk) % np);
    const int b = static_cast<int>(u / (static_cast<int64_t>(rblk) * np));
    int h = ps;
    if (a.head_idx) {
      if (a.H <= 32) {
        // the ps-th head (in index order) that no kept slot lists: lane s loads slot s's head
        const int32_t* hi = a.head_idx + static_cast<int64_t>(b) * a.head_idx_ld;
        const int hs = lane < a.H_kept ? hi[lane] : -1;
        const uint32_t kept = __reduce_or_sync(0xffffffffu, hs >= 0 && hs < 32 ? 1u << hs : 0u);
        uint32_t free_mask = ~kept & (a.H == 32 ? 0xffffffffu : (1u << a.H) - 1u);
        for (int k = 0; k < ps; ++k) free_mask &= free_mask - 1;
        h = free_mask ? __ffs(free_mask) - 1 : -1;
      } else {
        h = head_of_slot(a, b, a.H_kept + ps);
      }
    } else {
      h = a.H_kept + ps;
    }
    if (h < 0) continue;
    const int i0 = rb * kRows, rows = min(kRows, a.n_q - i0);
    for (int e = lane; e < rows * C8; e += 32) {
      const int i = i0 + e / C8, c8 = e % C8;
      *reinterpret_cast<uint4*>(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok + static_cast<int64_t>(h) * DH +
                                c8 * 8) = make_uint4(0, 0, 0, 0);
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(kMainThreads<DH>, 1) attn_main_kernel(AttnProblem p) {
  using C = MainCfg<DH>;
  constexpr int KT = C::KT;
  constexpr int NST = C::NST;
  const spatten_attn_args& a = p.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bars[M_N];
  __shared__ uint32_t tmem_base_s;
  __shared__ float colred[C::kT ? 1 : 2][2][4][C::kT ? 1 : KT];    // [tile parity][warpgroup][warp][key]
  __shared__ __align__(16) float nmb_s[2][128];   // transposed pass: -(m + log2 ell) of each query row
  __shared__ float hred[2][4];
  __shared__ uint32_t wcnt[8];
  __shared__ int abort_s;   // set when a role gave up waiting

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = p.n_pair * a.H_kept * a.B;
  const int n_tiles = (a.n_kv + KT - 1) / KT;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);

  if (warp == kMainMmaWarp<DH>) {
    tmem_alloc(&tmem_base_s, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    abort_s = 0;
    for (int qb = 0; qb < C::NQ; ++qb) {
      mbar_init(&bars[M_QF + qb], kMainProducers<DH>);
      mbar_init(&bars[M_QE + qb], 1);
    }
    mbar_init(&bars[M_OE], 256);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars[M_KF + s], kMainProducers<DH>);
      mbar_init(&bars[M_VF + s], kMainProducers<DH>);
      mbar_init(&bars[M_KE + s], 1);
      mbar_init(&bars[M_VE + s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&bars[M_SF + g], 1);
      mbar_init(&bars[M_SR + g], 128);
      mbar_init(&bars[M_PF + g], 128);
      mbar_init(&bars[M_PE + g], 1);
    }
    mbar_init(&bars[M_OD], 1);
    mbar_init(&bars[M_DR], 1);
    for (int s = 0; s < C::RS; ++s) {
      mbar_init(&bars[M_RF + s], 1);
      mbar_init(&bars[M_RE + s], kMainProducers<DH>);
    }
    fence_mbar_init();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;
  const uint32_t wlim = p.wait_limit;   // polls of one pipeline wait
  bool aborted = false;

  // item -> (sequence, kept head slot, pair)
  auto item_coords = [&](int it, int& b, int& slot, int& pair) {
    pair = it % p.n_pair;
    const int bs = it / p.n_pair;
    slot = bs % a.H_kept;
    b = bs / a.H_kept;
  };

  if (warp >= 8) {
    // warpgroups 2 and 3 (producers, MMA warp) give registers up to the softmax warpgroups; every
    // warp of a warpgroup executes this one instruction
    if constexpr (DH == 64) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp < kMainMmaWarp<DH>) {
      // ------------------------------------------------------------------------- producers
      const int ptid = tid - 256;
      uint32_t kc = 0, vc = 0, gjob = 0, qc = 0;
      constexpr int QCH = 256 * (DH / 8);   // 16-byte chunks of one item's query rows
      // the item's 256 query rows of its head, bf16, into query buffer qb at their swizzled fp16
      // positions (rows past n_q zero-filled); one commit group
      auto copy_q_async = [&](int item, uint32_t qbuf) {
        int b, slot, pair;
        item_coords(item, b, slot, pair);
        const int h = head_of_slot(a, b, slot);
        const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
        for (int e = ptid; e < QCH; e += kMainProducers<DH>) {
          const int rr = e / (DH / 8), c8 = e % (DH / 8), qi = pair * 256 + rr;
          const bool ok = qi < a.n_q;
          const __nv_bfloat16* src =
              ok ? q + (static_cast<int64_t>(b) * a.n_q + qi) * a.q_ld_tok + static_cast<int64_t>(h) * DH + c8 * 8 : q;
          cp_async16(smem + C::oQ + qbuf * 2 * C::QB + (rr >> 7) * C::QB + tile_off(rr & 127, c8, 128), src, ok ? 16u : 0u);
        }
        cp_async_commit();
      };
      // bf16 -> fp16 in place, each thread the chunks it copied
      auto convert_q_in_place = [&](uint32_t qbuf) {
        uint32_t mx = 0u;
        for (int e = ptid; e < QCH; e += kMainProducers<DH>) {
          const int rr = e / (DH / 8), c8 = e % (DH / 8);
          uint4* p = reinterpret_cast<uint4*>(smem + C::oQ + qbuf * 2 * C::QB + (rr >> 7) * C::QB + tile_off(rr & 127, c8, 128));
          const uint4 v = *p;
          mx = bf16x8_absmax(v, mx);
          *p = bf16x8_to_f16x8(v);
        }
        if (bf16_absmax_out_of_f16(mx)) report(a.dev_status, SPATTEN_E_RANGE);
      };
      uint32_t g_issued = 0, g_consumed = 0;   // staging-ring jobs issued / converted, whole kernel
      for (int it = blockIdx.x; it < n_items && !aborted; it += gridDim.x, ++qc) {
        int b, slot, pair;
        item_coords(it, b, slot, pair);
        const int h = head_of_slot(a, b, slot);
        const int64_t plane0 = (static_cast<int64_t>(b) * a.H + h) * a.kv_cap;
        const int32_t* kv_idx = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;
        JobStream<DH, KT, C::RS, kMainProducers<DH>> js{smem, C::oRaw, C::RAWB, &bars[M_RF], &bars[M_RE], &a, plane0, n_tiles, false, ptid,
                                    abort_flag, gjob};
        js.wlim = wlim;
        if (p.v_mask) js.vmask = p.v_mask + (static_cast<int64_t>(b) * a.H_kept + slot) * a.n_kv;
        struct Track {   // records the stream's progress however the item's loop is left
          JobStream<DH, KT, C::RS, kMainProducers<DH>>& js;
          uint32_t &gi, &gc;
          __device__ ~Track() { gi = js.g0 + js.issued; gc = js.g0 + js.consumed; }
        } track{js, g_issued, g_consumed};
        // the first raw key tiles start before the query tile (both in flight together)
        if (!kv_idx && ptid == 0 && !js.issue_ahead(0)) { aborted = true; break; }
        const uint32_t qb = qc % C::NQ;
        if constexpr (C::NQ == 2) {
          // this item's query tile was copied (bf16) into buffer qb during the previous item, or just
          // below for the first item: convert it in place to fp16 (each thread its own chunks)
          if (qc == 0) {
            if (!wait_bar(&bars[M_QE + qb], 1u, abort_flag, wlim)) { aborted = true; break; }
            copy_q_async(it, qb);
          }
          cp_async_wait_all();
          convert_q_in_place(qb);
          fence_async_smem();
          mbar_arrive(&bars[M_QF + qb]);
        } else {
          // query tile of the item once the previous item's score MMAs have read the buffer
          if (!wait_bar(&bars[M_QE], (qc & 1u) ^ 1u, abort_flag, wlim)) { aborted = true; break; }
          constexpr int NCH = 256 * (DH / 8);
          constexpr int BATCH = 8;
          const int i0 = pair * 256;
          const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
          uint32_t qmx = 0u;
          for (int e0 = ptid; e0 < NCH; e0 += BATCH * kMainProducers<DH>) {
            uint4 qv[BATCH];
  #pragma unroll
            for (int k = 0; k < BATCH; ++k) {
              const int e = e0 + k * kMainProducers<DH>;
              const int rr = e / (DH / 8), c8 = e % (DH / 8), qi = i0 + rr;
              qv[k] = make_uint4(0, 0, 0, 0);
              if (e < NCH && qi < a.n_q)
                qv[k] = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * a.n_q + qi) * a.q_ld_tok +
                                                             static_cast<int64_t>(h) * DH) + c8);
            }
  #pragma unroll
            for (int k = 0; k < BATCH; ++k) {
              const int e = e0 + k * kMainProducers<DH>;
              const int rr = e / (DH / 8), c8 = e % (DH / 8);
              if (e < NCH) {
                qmx = bf16x8_absmax(qv[k], qmx);
                *reinterpret_cast<uint4*>(smem + C::oQ + (rr >> 7) * C::QB + tile_off(rr & 127, c8, 128)) =
                    bf16x8_to_f16x8(qv[k]);
              }
            }
          }
          if (bf16_absmax_out_of_f16(qmx)) report(a.dev_status, SPATTEN_E_RANGE);
          fence_async_smem();
          mbar_arrive(&bars[M_QF]);
        }
        // pass A keys, then pass B keys and values
        for (int j = 0; j < 3 * n_tiles; ++j) {
          if constexpr (C::NQ == 2) {
            // at the first pass-B job the previous item is done with the other query buffer: copy
            // the next item's query rows into it
            if (j == n_tiles && it + static_cast<int>(gridDim.x) < n_items) {
              const uint32_t nb = (qc + 1) % C::NQ;
              if (!wait_bar(&bars[M_QE + nb], (((qc + 1) / C::NQ) & 1u) ^ 1u, abort_flag, wlim)) { aborted = true; break; }
              copy_q_async(it + static_cast<int>(gridDim.x), nb);
            }
          }
          if (!kv_idx && ptid == 0 && !js.issue_ahead(j)) { aborted = true; break; }
          bool is_v;
          int t;
          js.job(j, is_v, t);
          uint32_t& cnt = is_v ? vc : kc;
          const uint32_t st = cnt % NST;
          if (!wait_bar(&bars[(is_v ? M_VE : M_KE) + st], ((cnt / NST) & 1u) ^ 1u, abort_flag, wlim)) { aborted = true; break; }
          if (!js.convert(j, (is_v ? C::oV : C::oK) + st * C::TB, kv_idx)) { aborted = true; break; }
          mbar_arrive(&bars[(is_v ? M_VF : M_KF) + st]);
          ++cnt;
        }
        gjob += 3 * n_tiles;
      }
      cp_async_wait_all();   // no query copy may land after the CTA has left
      if (aborted && ptid == 0)   // bulk copies already armed complete before shared memory is released
        for (uint32_t gj = g_consumed; gj < g_issued; ++gj) drain_wait(&bars[M_RF + gj % C::RS], (gj / C::RS) & 1u);
    } else {
      // ------------------------------------------------------------------------- MMA issue
      if (lane == 0) {
        uint32_t kc = 0, vc = 0, sc[2] = {0, 0}, pc[2] = {0, 0}, ic = 0;
        uint32_t sQ0 = smem_u32(smem + C::oQ), sQ1 = smem_u32(smem + C::oQ + C::QB);
        // scores of one key tile for both warpgroups: S = Q K^T (pass A, and pass B in row
        // orientation) or S^T = K Q^T (pass B, transposed)
        auto qk_both = [&](bool trans) -> bool {
          const uint32_t ks = kc % NST;
          if (!wait_bar(&bars[M_KF + ks], (kc / NST) & 1u, abort_flag, wlim)) return false;
          const uint32_t sK = smem_u32(smem + C::oK + ks * C::TB);
          if (!wait_bar(&bars[M_SR + 0], (sc[0] & 1u) ^ 1u, abort_flag, wlim)) return false;
          tc_after_sync();
          if (C::kT && trans) mma_kq<DH, KT>(tmem + C::tS, sK, sQ0);
          else mma_qk<DH, KT>(tmem + C::tS, sQ0, sK, 0);
          mma_commit(&bars[M_SF + 0]);
          ++sc[0];
          if (!wait_bar(&bars[M_SR + 1], (sc[1] & 1u) ^ 1u, abort_flag, wlim)) return false;
          tc_after_sync();
          if (C::kT && trans) mma_kq<DH, KT>(tmem + C::tS + KT, sK, sQ1);
          else mma_qk<DH, KT>(tmem + C::tS + KT, sQ1, sK, 0);
          mma_commit(&bars[M_SF + 1]);
          ++sc[1];
          mma_commit(&bars[M_KE + ks]);
          ++kc;
          return true;
        };
        for (int it = blockIdx.x; it < n_items && !aborted; it += gridDim.x, ++ic) {
          const uint32_t qb = ic % C::NQ;
          sQ0 = smem_u32(smem + C::oQ + qb * 2 * C::QB);
          sQ1 = sQ0 + C::QB;
          if (!wait_bar(&bars[M_QF + qb], (ic / C::NQ) & 1u, abort_flag, wlim)) { aborted = true; break; }
          for (int t = 0; t < n_tiles && !aborted; ++t)   // pass A
            if (!qk_both(false)) aborted = true;
          if (aborted) break;
          if (!qk_both(true)) { aborted = true; break; }   // pass B, tile 0
          if (n_tiles == 1) mma_commit(&bars[M_QE + qb]);  // the item's last read of Q is issued
          // the previous item's O must have been read before this item's first P V overwrites it
          if (!wait_bar(&bars[M_OE], (ic & 1u) ^ 1u, abort_flag, wlim)) { aborted = true; break; }
          for (int t = 0; t < n_tiles && !aborted; ++t) {
            if (t + 1 < n_tiles) {
              if (!qk_both(true)) { aborted = true; break; }
              if (t + 2 == n_tiles) mma_commit(&bars[M_QE + qb]);
            }
            const uint32_t vs = vc % NST;
            if (!wait_bar(&bars[M_VF + vs], (vc / NST) & 1u, abort_flag, wlim)) { aborted = true; break; }
            const uint32_t sV = smem_u32(smem + C::oV + vs * C::TB);
            for (int gg = 0; gg < 2 && !aborted; ++gg) {
              if (!wait_bar(&bars[M_PF + gg], pc[gg] & 1u, abort_flag, wlim)) { aborted = true; break; }
              tc_after_sync();
              if constexpr (C::kT)
                mma_pv_mn<DH, KT>(tmem + C::tO + gg * DH, smem_u32(smem + C::oP + gg * C::PB), sV, t > 0 ? 1u : 0u);
              else
                mma_pv<DH, KT>(tmem + C::tO + gg * DH, smem_u32(smem + C::oP + gg * C::PB), sV, t > 0 ? 1u : 0u);
              mma_commit(&bars[M_PE + gg]);
              ++pc[gg];
            }
            if (aborted) break;
            mma_commit(&bars[M_VE + vs]);
            ++vc;
          }
          if (!aborted) mma_commit(&bars[M_OD]);
        }
      }
    }
  } else {
    if constexpr (DH == 64) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------------------------------------------------------------------- softmax
    if (a.zero_pruned_heads && a.H_kept < a.H) zero_pruned_share<DH>(a, o, warp, lane);
    const int g = warp >> 2;                        // warpgroup
    const int r = tid & 127;                        // row within the warpgroup's tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t sc = 0, pc = 0, oc = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++oc) {
      if (!softmax_all(!aborted)) { aborted = true; break; }   // both warpgroups start the item together
      int b, slot, pair;
      item_coords(it, b, slot, pair);
      const int h = head_of_slot(a, b, slot);
      const int64_t bh = static_cast<int64_t>(b) * a.H + h;
      const int i = pair * 256 + g * 128 + r;
      const bool row_ok = i < a.n_q;
      const float c2 = a.k_scale[bh] * a.sm_scale * kLog2e;
      const int64_t list_base = (static_cast<int64_t>(b) * a.H_kept + slot) * p.n_pair + pair;
      float m2 = -INFINITY, l = 0.0f;

      // ---- pass A: MSB statistics
      for (int t = 0; t < n_tiles; ++t) {
        if (!__all_sync(0xffffffffu, wait_bar(&bars[M_SF + g], sc & 1u, abort_flag, wlim))) { aborted = true; break; }
        tc_after_sync();
#pragma unroll 1
        for (int hh = 0; hh < KT / 64; ++hh) {
          float v[64];
          __syncwarp();
          tmem_ld32(tmem + lane_base + C::tS + g * KT + hh * 64, v);
          tmem_ld32(tmem + lane_base + C::tS + g * KT + hh * 64 + 32, v + 32);
          tmem_ld_wait();
          if (hh == KT / 64 - 1) {
            tc_before_sync();
            mbar_arrive(&bars[M_SR + g]);
          }
          if (t * KT + hh * 64 + 64 <= a.n_kv) {   // a full chunk (uniform over the CTA)
            stats64_scaled(v, c2, m2, l);
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = (t * KT + hh * 64 + j < a.n_kv) ? v[j] * c2 : -INFINITY;
            stats64(v, m2, l);
          }
        }
        ++sc;
      }
      const bool flag = !aborted && row_ok && (1.0f / l < a.refetch_threshold);
      // p = 2^(c2 s - m2) / ell = 2^(c2 s + nmb); rows that are not stored here get p = 0
      if constexpr (C::kT) nmb_s[g][r] = (row_ok && !flag) ? -(m2 + log2f(l)) : -INFINITY;

      // ---- flagged rows -> packed list (ascending row ids); counts of the item
      const unsigned bal = __ballot_sync(0xffffffffu, flag);
      if (lane == 0) wcnt[warp] = __popc(bal);
      if (!softmax_all(!aborted)) { aborted = true; break; }
      {
        uint32_t pos = __popc(bal & ((1u << lane) - 1u)), total = 0;
        for (int w = 0; w < 8; ++w) {
          if (w < warp) pos += wcnt[w];
          total += wcnt[w];
        }
        if (flag) p.flag_list[list_base * 256 + pos] = i;
        if (tid == 0) p.flag_cnt[list_base] = static_cast<int32_t>(total);
        if (tid == 0 && total && a.refetch_count) atomicAdd(a.refetch_count, static_cast<int>(total));
      }

      // ---- pass B: probabilities of the unflagged rows, column sums, P V
      if constexpr (C::kT) {
        // transposed: S^T = K Q^T puts one key on each TMEM lane; thread r owns key t*KT + r and
        // sees the warpgroup's 128 query rows as columns, so its column sum of P is a register
        // accumulation and it writes its key's column of P (MN-major: rows contiguous)
        uint8_t* Pt = smem + C::oP + g * C::PB;
        const int qt128 = pair * 2 + g;
        const int64_t part_row = ((static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt128) * a.n_kv;
        const float4* nmb4 = reinterpret_cast<const float4*>(&nmb_s[g][0]);
        const float2 c2x2 = make_float2(c2, c2);
        const uint32_t kcol = (static_cast<uint32_t>(r) >> 3) * 1024u + (static_cast<uint32_t>(r) & 7u) * 128u;
        for (int t = 0; t < n_tiles; ++t) {
          if (!wg_all(wait_bar(&bars[M_SF + g], sc & 1u, abort_flag, wlim), 1 + g)) { aborted = true; break; }
          tc_after_sync();
          const int key = t * KT + r;
          const bool key_ok = key < a.n_kv;
          float2 cs0 = make_float2(0.0f, 0.0f), cs1 = cs0;
          // two halves of 64 query rows: the TMEM columns are released once the second half is
          // loaded, half a tile before the probabilities are done
#pragma unroll 1
          for (int hf = 0; hf < 2; ++hf) {
            float v[64];
            __syncwarp();
            tmem_ld32(tmem + lane_base + C::tS + g * KT + hf * 64, v);
            tmem_ld32(tmem + lane_base + C::tS + g * KT + hf * 64 + 32, v + 32);
            tmem_ld_wait();
            if (hf == 1) {
              tc_before_sync();
              mbar_arrive(&bars[M_SR + g]);
              ++sc;
            } else if (!wg_all(wait_bar(&bars[M_PE + g], (pc & 1u) ^ 1u, abort_flag, wlim), 1 + g)) {
              // the previous tile's P V must be done before this tile's P overwrites the buffer
              aborted = true;
              break;
            }
            if (key_ok) {
#pragma unroll
              for (int c = 0; c < 8; ++c) {   // query rows 64 hf + 8c .. + 7
                const float4 na = nmb4[16 * hf + 2 * c], nb = nmb4[16 * hf + 2 * c + 1];
                float2 e0 = ffma2(make_float2(v[8 * c + 0], v[8 * c + 1]), c2x2, make_float2(na.x, na.y));
                float2 e1 = ffma2(make_float2(v[8 * c + 2], v[8 * c + 3]), c2x2, make_float2(na.z, na.w));
                float2 e2 = ffma2(make_float2(v[8 * c + 4], v[8 * c + 5]), c2x2, make_float2(nb.x, nb.y));
                float2 e3 = ffma2(make_float2(v[8 * c + 6], v[8 * c + 7]), c2x2, make_float2(nb.z, nb.w));
                e0 = exp2_pair<0>(e0);
                e1 = exp2_pair<1>(e1);
                e2 = exp2_pair<2>(e2);
                e3 = exp2_pair<3>(e3);
                cs0 = fadd2(cs0, e0);
                cs1 = fadd2(cs1, e1);
                cs0 = fadd2(cs0, e2);
                cs1 = fadd2(cs1, e3);
                *reinterpret_cast<uint4*>(Pt + hf * (KT * 128u) + kcol + ((static_cast<uint32_t>(c) ^ (r & 7u)) << 4)) =
                    make_uint4(pack_f16x2(e0.x, e0.y), pack_f16x2(e1.x, e1.y), pack_f16x2(e2.x, e2.y),
                               pack_f16x2(e3.x, e3.y));
              }
            } else {   // keys past the end: zero columns (their V rows are zero-filled too)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(Pt + hf * (KT * 128u) + kcol + ((static_cast<uint32_t>(c) ^ (r & 7u)) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
          }
          if (aborted) break;   // uniform over the warpgroup
          fence_async_smem();
          mbar_arrive(&bars[M_PF + g]);
          ++pc;
          if (key < a.n_kv && qt128 < p.n_qt) p.tok_part[part_row + key] = (cs0.x + cs1.x) + (cs0.y + cs1.y);
        }
      } else {
        const bool live = row_ok && !flag;
        // p = 2^(c2 s - m2) / ell = 2^(c2 s - mb); rows that are not stored here get p = 0
        const float mb = live ? m2 + log2f(l) : INFINITY;
        uint8_t* Pt = smem + C::oP + g * C::PB;
        const int qt128 = pair * 2 + g;
        const int64_t part_row = ((static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt128) * a.n_kv;
        for (int t = 0; t < n_tiles; ++t) {
          if (!wg_all(wait_bar(&bars[M_SF + g], sc & 1u, abort_flag, wlim), 1 + g)) { aborted = true; break; }
          tc_after_sync();
#pragma unroll 1
          for (int hh = 0; hh < KT / 64; ++hh) {
            float v[32], w[32];
            __syncwarp();
            tmem_ld32(tmem + lane_base + C::tS + g * KT + hh * 64, v);
            tmem_ld32(tmem + lane_base + C::tS + g * KT + hh * 64 + 32, w);
            tmem_ld_wait();
            if (hh == KT / 64 - 1) {
              tc_before_sync();
              mbar_arrive(&bars[M_SR + g]);
            }
            // the previous tile's P V must be done before this tile's P overwrites the buffer; the
            // score load and the exponentials below overlap it
            if (hh == 0 && !wg_all(wait_bar(&bars[M_PE + g], (pc & 1u) ^ 1u, abort_flag, wlim), 1 + g)) {
              aborted = true;
              break;
            }
            const int kb = t * KT + hh * 64;
            if (kb + 64 <= a.n_kv) {   // a full chunk (uniform over the CTA)
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                v[j] = ex2(fmaf(v[j], c2, -mb));
                w[j] = ex2(fmaf(w[j], c2, -mb));
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                v[j] = kb + j < a.n_kv ? ex2(fmaf(v[j], c2, -mb)) : 0.0f;
                w[j] = kb + 32 + j < a.n_kv ? ex2(fmaf(w[j], c2, -mb)) : 0.0f;
              }
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              *reinterpret_cast<uint4*>(Pt + tile_off(r, hh * 8 + q4, 128)) =
                  make_uint4(pack_f16x2(v[8 * q4 + 0], v[8 * q4 + 1]), pack_f16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                             pack_f16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_f16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
              *reinterpret_cast<uint4*>(Pt + tile_off(r, hh * 8 + 4 + q4, 128)) =
                  make_uint4(pack_f16x2(w[8 * q4 + 0], w[8 * q4 + 1]), pack_f16x2(w[8 * q4 + 2], w[8 * q4 + 3]),
                             pack_f16x2(w[8 * q4 + 4], w[8 * q4 + 5]), pack_f16x2(w[8 * q4 + 6], w[8 * q4 + 7]));
            }
            float sv, sw;
            warp_colsum32x2(v, w, sv, sw);
            colred[t & 1][g][warp & 3][hh * 64 + lane] = sv;
            colred[t & 1][g][warp & 3][hh * 64 + 32 + lane] = sw;
          }
          if (aborted) break;   // uniform over the warpgroup
          ++sc;
          fence_async_smem();
          mbar_arrive(&bars[M_PF + g]);
          ++pc;
          named_sync(1 + g, 128);
          if (r < KT) {
            const int key = t * KT + r;
            if (key < a.n_kv && qt128 < p.n_qt)
              p.tok_part[part_row + key] = ((colred[t & 1][g][0][r] + colred[t & 1][g][1][r]) + colred[t & 1][g][2][r]) +
                                           colred[t & 1][g][3][r];
          }
        }
      }

      // ---- epilogue: O of the unflagged rows, head importance partial, refetch flags
      float habs = 0.0f;
      if (!aborted) {
        if (!wg_all(wait_bar(&bars[M_OD], oc & 1u, abort_flag, wlim), 1 + g)) aborted = true;
      }
      if (!aborted) {
        tc_after_sync();
        float ov[DH];
#pragma unroll
        for (int ch = 0; ch < DH / 32; ++ch) tmem_ld32(tmem + lane_base + C::tO + g * DH + ch * 32, ov + ch * 32);
        tmem_ld_wait();
        tc_before_sync();
        mbar_arrive(&bars[M_OE]);   // the next item's P V may overwrite O
        const float vs = a.v_scale[bh];
        if (row_ok && !flag) {
#pragma unroll
          for (int ch = 0; ch < DH / 32; ++ch)
            store_o_row(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok + static_cast<int64_t>(h) * DH + ch * 32,
                        ov + ch * 32, vs, habs);
        }
        if (row_ok && a.refetch_flags) a.refetch_flags[bh * a.refetch_flags_ld + i] = flag ? 1 : 0;
      }
      habs = warp_sum(habs);
      if (lane == 0) hred[g][warp & 3] = habs;
      if (!softmax_all(!aborted)) { aborted = true; break; }
      if (tid == 0 || tid == 128) {
        const int qt128 = pair * 2 + (tid >> 7);
        if (qt128 < p.n_qt)
          p.head_part[(static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt128] =
              ((hred[tid >> 7][0] + hred[tid >> 7][1]) + hred[tid >> 7][2]) + hred[tid >> 7][3];
      }
    }
  }
  const bool any_abort = __syncthreads_or(aborted);
  if (any_abort && tid == 0) report(a.dev_status, SPATTEN_E_TIMEOUT);
  // after an abort no flagged-row list of this CTA's items is valid: their counts become 0, so
  // that the refetch and reduce kernels read none of them (item it's list is entry it)
  if (any_abort && p.flag_cnt)
    for (int64_t it = blockIdx.x + static_cast<int64_t>(tid) * gridDim.x; it < n_items;
         it += static_cast<int64_t>(gridDim.x) * blockDim.x)
      p.flag_cnt[it] = 0;
  if (any_abort && warp == kMainMmaWarp<DH> && lane == 0) {   // every MMA already issued completes before TMEM is freed
    mma_commit(&bars[M_DR]);
    drain_wait(&bars[M_DR], 0u);
  }
  tc_before_sync();
  __syncthreads();
  if (warp == kMainMmaWarp<DH>) {
    tc_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// =================================================================================================
// FULL kernel: packed flagged rows at full precision
// =================================================================================================
template <int DH>
struct FullCfg {
  // 64-key tiles: two CTAs of d_h 64 fit one SM (shared memory and tensor memory), so that two
  // heads' producers and softmax warps overlap
  static constexpr int KT = 64;
  static constexpr uint32_t kTmem = 256;         // S (2 x KT columns) and O (DH columns)
  static constexpr uint32_t QB = 128u * DH * 2u;
  static constexpr uint32_t TB = static_cast<uint32_t>(KT) * DH * 2u;
  static constexpr uint32_t PB = 128u * KT * 2u;
  static constexpr int RS = 3;                   // raw (MSB + LSB) tiles in flight
  static constexpr uint32_t RAWB = static_cast<uint32_t>(KT) * DH * 3u / 2u;
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = QB;             // 2 stages of one combined (16·MSB + LSB) tile
  static constexpr uint32_t oV = oK + 2 * TB;    // 2 stages of one combined tile
  static constexpr uint32_t oP = oV + 2 * TB;    // 1 buffer
  static constexpr uint32_t oRaw = oP + PB;      // RS staging slots
  static constexpr uint32_t kSmem = oRaw + RS * RAWB + 1024u;
  static constexpr uint32_t tS = 0;              // + buffer * KT
  static constexpr uint32_t tO = 2u * KT;
};

enum : int { F_Q = 0, F_KF = 1, F_KE = 3, F_VF = 5, F_VE = 7, F_SF = 9, F_SR = 11, F_PF = 13, F_PE = 15, F_OD = 17,
             F_RF = 18, F_RE = 21, F_DR = 24, F_N = 25 };
constexpr int kMaxPairs = 256;   // query rows per head up to 256 * 256

template <int DH>
__global__ void __launch_bounds__(256, DH == 64 ? 2 : 1) attn_full_kernel(AttnProblem p) {
  using C = FullCfg<DH>;
  constexpr int KT = C::KT;
  const spatten_attn_args& a = p.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bars[F_N];
  __shared__ uint32_t tmem_base_s;
  __shared__ float colred[2][4][KT];
  __shared__ float hred[4];
  __shared__ int abort_s;   // set when a role gave up waiting
  __shared__ int pref[kMaxPairs + 1];
  __shared__ int rows[128];

  // the flagged rows of the head, concatenated over its 256-row pair tiles in order; this CTA
  // takes packed rows [128u, 128u + 128)
  const int u = blockIdx.x, slot = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t head_lists = (static_cast<int64_t>(b) * a.H_kept + slot) * p.n_pair;
  if (tid == 0) {
    int acc = 0;
    for (int pp = 0; pp < p.n_pair; ++pp) {
      pref[pp] = acc;
      acc += p.flag_cnt[head_lists + pp];
    }
    pref[p.n_pair] = acc;
  }
  __syncthreads();
  const int rows_here = min(128, pref[p.n_pair] - u * 128);
  if (rows_here <= 0) return;   // uniform: nothing to recompute in this packed tile
  if (tid < rows_here) {
    const int k = u * 128 + tid;
    int pp = 0;
    while (pref[pp + 1] <= k) ++pp;
    rows[tid] = p.flag_list[(head_lists + pp) * 256 + (k - pref[pp])];
  }

  const int h = head_of_slot(a, b, slot);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);

  if (warp == 7) {
    tmem_alloc(&tmem_base_s, C::kTmem);
    tmem_relinquish();
  }
  if (tid == 0) {
    abort_s = 0;
    mbar_init(&bars[F_Q], 224);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[F_KF + s], kProducerThreads);
      mbar_init(&bars[F_VF + s], kProducerThreads);
      mbar_init(&bars[F_KE + s], 1);
      mbar_init(&bars[F_VE + s], 1);
      mbar_init(&bars[F_SF + s], 1);
      mbar_init(&bars[F_SR + s], 128);
      mbar_init(&bars[F_PF + s], 128);
      mbar_init(&bars[F_PE + s], 1);
    }
    mbar_init(&bars[F_OD], 1);
    mbar_init(&bars[F_DR], 1);
    for (int s = 0; s < C::RS; ++s) {
      mbar_init(&bars[F_RF + s], 1);
      mbar_init(&bars[F_RE + s], kProducerThreads);
    }
    fence_mbar_init();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;
  const uint32_t wlim = p.wait_limit;   // polls of one pipeline wait

  const int64_t bh = static_cast<int64_t>(b) * a.H + h;
  const int64_t plane0 = bh * a.kv_cap;
  const int32_t* kv_idx = a.kv_idx ? a.kv_idx + static_cast<int64_t>(b) * a.kv_idx_ld : nullptr;
  const int n_tiles = (a.n_kv + KT - 1) / KT;
  bool aborted = false;

  const int r = tid;                      // softmax: packed row r
  const bool row_ok = tid < 128 && r < rows_here;
  const int i = row_ok ? rows[r] : 0;
  const bool warp_live = warp < 4 && warp * 32 < rows_here;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const float c2 = a.k_scale[bh] * a.sm_scale * kLog2e;
  float m2 = -INFINITY, l = 0.0f;

  if (warp != 7) {
    // gathered Q rows: every thread but the MMA warp, all of its loads in flight at once
    constexpr int NCH = 128 * (DH / 8);
    constexpr int PER = (NCH + 223) / 224;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
    uint4 qv[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = tid + k * 224;
      const int rr = e / (DH / 8), c8 = e % (DH / 8);
      qv[k] = make_uint4(0, 0, 0, 0);
      if (e < NCH && rr < rows_here)
        qv[k] = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(b) * a.n_q + rows[rr]) * a.q_ld_tok +
                                                     static_cast<int64_t>(h) * DH) + c8);
    }
    uint32_t qmx = 0u;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = tid + k * 224;
      const int rr = e / (DH / 8), c8 = e % (DH / 8);
      if (e < NCH) {
        qmx = bf16x8_absmax(qv[k], qmx);
        *reinterpret_cast<uint4*>(smem + C::oQ + tile_off(rr, c8, 128)) = bf16x8_to_f16x8(qv[k]);
      }
    }
    if (bf16_absmax_out_of_f16(qmx)) report(a.dev_status, SPATTEN_E_RANGE);
    fence_async_smem();
    mbar_arrive(&bars[F_Q]);
  }
  if (warp >= 4 && warp < 7) {
    // ------------------------------------------------------------------------- producers
    const int ptid = tid - 128;
    JobStream<DH, KT, C::RS, kProducerThreads> js{smem, C::oRaw, C::RAWB, &bars[F_RF], &bars[F_RE], &a, plane0, n_tiles, true, ptid,
                                abort_flag};
    js.wlim = wlim;
    if (p.v_mask) js.vmask = p.v_mask + (static_cast<int64_t>(b) * a.H_kept + slot) * a.n_kv;
    uint32_t kc = 0, vc = 0;
    auto run_jobs = [&](int j0, int j1) {
      for (int j = j0; j < j1; ++j) {
        if (!kv_idx && ptid == 0 && !js.issue_ahead(j)) { aborted = true; return; }
        bool is_v;
        int t;
        js.job(j, is_v, t);
        uint32_t& cnt = is_v ? vc : kc;
        const uint32_t st = cnt & 1u;
        if (!wait_bar(&bars[(is_v ? F_VE : F_KE) + st], ((cnt >> 1) & 1u) ^ 1u, abort_flag, wlim)) { aborted = true; return; }
        if (!js.convert(j, (is_v ? C::oV : C::oK) + st * C::TB, kv_idx)) { aborted = true; return; }
        mbar_arrive(&bars[(is_v ? F_VF : F_KF) + st]);
        ++cnt;
      }
    };
    run_jobs(0, 3 * n_tiles);   // pass A keys, then pass B keys and values, without a block barrier
    if (ptid == 0)   // after an abort: bulk copies already armed complete before shared memory is released
      for (uint32_t gj = js.consumed; gj < js.issued; ++gj) drain_wait(&bars[F_RF + gj % C::RS], (gj / C::RS) & 1u);
  } else if (warp == 7) {
    // ------------------------------------------------------------------------- MMA issue
    uint32_t kc = 0, vc = 0, sc[2] = {0, 0}, pc[2] = {0, 0};
    const uint32_t sQ = smem_u32(smem + C::oQ);
    auto qk = [&](int t) -> bool {
      const uint32_t ks = kc & 1u;
      if (!wait_bar(&bars[F_KF + ks], (kc >> 1) & 1u, abort_flag, wlim)) return false;
      const int sb = t & 1;
      if (!wait_bar(&bars[F_SR + sb], (sc[sb] & 1u) ^ 1u, abort_flag, wlim)) return false;
      tc_after_sync();
      const uint32_t sK = smem_u32(smem + C::oK + ks * C::TB);
      mma_qk<DH, KT>(tmem + C::tS + sb * KT, sQ, sK, 0);   // the combined (16·MSB + LSB) tile
      mma_commit(&bars[F_SF + sb]);
      mma_commit(&bars[F_KE + ks]);
      ++sc[sb];
      ++kc;
      return true;
    };
    if (lane == 0) {
      if (!wait_bar(&bars[F_Q], 0, abort_flag, wlim)) aborted = true;
      for (int t = 0; t < n_tiles && !aborted; ++t)
        if (!qk(t)) aborted = true;
    }
    if (lane == 0 && !aborted) {   // pass B follows at once
      if (!qk(0)) aborted = true;
      for (int t = 0; t < n_tiles && !aborted; ++t) {
        if (t + 1 < n_tiles && !qk(t + 1)) { aborted = true; break; }
        const int pb = 0;   // single P buffer
        if (!wait_bar(&bars[F_PF + pb], pc[pb] & 1u, abort_flag, wlim)) { aborted = true; break; }
        const uint32_t vs = vc & 1u;
        if (!wait_bar(&bars[F_VF + vs], (vc >> 1) & 1u, abort_flag, wlim)) { aborted = true; break; }
        tc_after_sync();
        const uint32_t sP = smem_u32(smem + C::oP + pb * C::PB);
        const uint32_t sV = smem_u32(smem + C::oV + vs * C::TB);
        mma_pv<DH, KT>(tmem + C::tO, sP, sV, t > 0 ? 1u : 0u);   // the combined tile
        mma_commit(&bars[F_PE + pb]);
        mma_commit(&bars[F_VE + vs]);
        ++pc[pb];
        ++vc;
      }
      if (!aborted) mma_commit(&bars[F_OD]);
    }
  } else {
    // ------------------------------------------------------------------------- softmax (pass A)
    uint32_t sc[2] = {0, 0};
    for (int t = 0; t < n_tiles; ++t) {
      const int sb = t & 1;
      if (!__all_sync(0xffffffffu, wait_bar(&bars[F_SF + sb], sc[sb] & 1u, abort_flag, wlim))) { aborted = true; break; }
      tc_after_sync();
      if (warp_live) {
#pragma unroll 1
        for (int hh = 0; hh < KT / 64; ++hh) {
          float v[64];
          __syncwarp();
          tmem_ld32(tmem + lane_base + C::tS + sb * KT + hh * 64, v);
          tmem_ld32(tmem + lane_base + C::tS + sb * KT + hh * 64 + 32, v + 32);
          tmem_ld_wait();
          if (t * KT + hh * 64 + 64 <= a.n_kv) {   // a full chunk
            stats64_scaled(v, c2, m2, l);
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = (t * KT + hh * 64 + j < a.n_kv) ? v[j] * c2 : -INFINITY;
            stats64(v, m2, l);
          }
        }
      }
      tc_before_sync();
      mbar_arrive(&bars[F_SR + sb]);
      ++sc[sb];
    }
    aborted = !wg_all(!aborted, 1);   // the warpgroup enters pass B together
    // ------------------------------------------------------------------------- softmax (pass B)
    if (!aborted) {
      uint32_t pc[2] = {0, 0};
      const float mb = row_ok ? m2 + log2f(l) : INFINITY;   // p = 2^(c2 s - mb)
      const int64_t part_row = ((static_cast<int64_t>(b) * a.H_kept + slot) * 2 * p.n_pair + u) * a.n_kv;
      for (int t = 0; t < n_tiles; ++t) {
        const int sb = t & 1;
        const int pb = 0;   // single P buffer
        if (!wg_all(wait_bar(&bars[F_PE + pb], (pc[pb] & 1u) ^ 1u, abort_flag, wlim), 1)) { aborted = true; break; }
        if (!wg_all(wait_bar(&bars[F_SF + sb], sc[sb] & 1u, abort_flag, wlim), 1)) { aborted = true; break; }
        tc_after_sync();
        uint8_t* Pt = smem + C::oP + pb * C::PB;
#pragma unroll 1
        for (int hh = 0; hh < KT / 64; ++hh) {
          float v[32], w[32];
          if (warp_live) {
            __syncwarp();
            tmem_ld32(tmem + lane_base + C::tS + sb * KT + hh * 64, v);
            tmem_ld32(tmem + lane_base + C::tS + sb * KT + hh * 64 + 32, w);
            tmem_ld_wait();
            const int kb = t * KT + hh * 64;
            if (kb + 64 <= a.n_kv) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                v[j] = ex2(fmaf(v[j], c2, -mb));
                w[j] = ex2(fmaf(w[j], c2, -mb));
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                v[j] = kb + j < a.n_kv ? ex2(fmaf(v[j], c2, -mb)) : 0.0f;
                w[j] = kb + 32 + j < a.n_kv ? ex2(fmaf(w[j], c2, -mb)) : 0.0f;
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = w[j] = 0.0f;
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            *reinterpret_cast<uint4*>(Pt + tile_off(r, hh * 8 + q4, 128)) =
                make_uint4(pack_f16x2(v[8 * q4 + 0], v[8 * q4 + 1]), pack_f16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                           pack_f16x2(v[8 * q4 + 4], v[8 * q4 + 5]), pack_f16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
            *reinterpret_cast<uint4*>(Pt + tile_off(r, hh * 8 + 4 + q4, 128)) =
                make_uint4(pack_f16x2(w[8 * q4 + 0], w[8 * q4 + 1]), pack_f16x2(w[8 * q4 + 2], w[8 * q4 + 3]),
                           pack_f16x2(w[8 * q4 + 4], w[8 * q4 + 5]), pack_f16x2(w[8 * q4 + 6], w[8 * q4 + 7]));
          }
          float sv = 0.0f, sw = 0.0f;
          if (warp_live) warp_colsum32x2(v, w, sv, sw);
          colred[t & 1][warp][hh * 64 + lane] = sv;
          colred[t & 1][warp][hh * 64 + 32 + lane] = sw;
        }
        tc_before_sync();
        mbar_arrive(&bars[F_SR + sb]);
        ++sc[sb];
        fence_async_smem();
        mbar_arrive(&bars[F_PF + pb]);
        ++pc[pb];
        named_sync(1, 128);
        if (r < KT) {
          const int key = t * KT + r;
          if (key < a.n_kv)
            p.full_part[part_row + key] = ((colred[t & 1][0][r] + colred[t & 1][1][r]) + colred[t & 1][2][r]) + colred[t & 1][3][r];
        }
      }
    }
  }

  // ------------------------------------------------------------------------- epilogue
  float habs = 0.0f;
  if (warp < 4 && !aborted) {
    if (!wait_bar(&bars[F_OD], 0, abort_flag, wlim)) aborted = true;
    aborted = __any_sync(0xffffffffu, aborted);   // warp-uniform before the TMEM loads
    tc_after_sync();
    if (!aborted && warp_live) {
      const float vs = a.v_scale[bh];
#pragma unroll 1
      for (int ch = 0; ch < DH / 32; ++ch) {
        float v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_base + C::tO + ch * 32, v);
        tmem_ld_wait();
        if (row_ok)
          store_o_row(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok + static_cast<int64_t>(h) * DH + ch * 32, v,
                      vs, habs);
      }
    }
  }
  if (warp < 4) {
    habs = warp_sum(habs);
    if (lane == 0) hred[warp] = habs;
  }
  if (__syncthreads_or(aborted)) aborted = true;
  if (aborted && warp == 7 && lane == 0) {   // every MMA already issued completes before TMEM is freed
    mma_commit(&bars[F_DR]);
    drain_wait(&bars[F_DR], 0u);
  }
  if (tid == 0) {
    p.full_head[(static_cast<int64_t>(b) * a.H_kept + slot) * 2 * p.n_pair + u] = ((hred[0] + hred[1]) + hred[2]) + hred[3];
    if (aborted) report(a.dev_status, SPATTEN_E_TIMEOUT);
  }
  tc_before_sync();
  __syncthreads();
  if (warp == 7) {
    tc_after_sync();
    tmem_dealloc(tmem, C::kTmem);
  }
}

template <int DH>
int32_t launch(const AttnProblem& p, cudaStream_t st) {
  static DeviceOnce once;
  int dev = 0;
  SPT_TRY(once_per_device(once, &dev, [](int) -> int32_t {
    // the register split waits, without a bound, for registers the block holds: launch only when
    // the block's registers at launch cover it
    cudaFuncAttributes fa{};
    SPT_CUDA(cudaFuncGetAttributes(&fa, attn_main_kernel<DH>));
    if (DH == 64 && static_cast<int64_t>(fa.numRegs) * kMainThreads<DH> < 256LL * kSoftmaxRegs + 256LL * kOtherRegs)
      return SPATTEN_E_UNSUPPORTED;
    SPT_CUDA(cudaFuncSetAttribute(attn_main_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(MainCfg<DH>::kSmem)));
    SPT_CUDA(cudaFuncSetAttribute(attn_full_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(FullCfg<DH>::kSmem)));
    return SPATTEN_OK;
  }));
  const int64_t items = static_cast<int64_t>(p.n_pair) * p.a.H_kept * p.a.B;
  const int grid = static_cast<int>(std::min<int64_t>(items, sm_count()));
  attn_main_kernel<DH><<<grid, kMainThreads<DH>, MainCfg<DH>::kSmem, st>>>(p);
  SPT_TRY(launch_status());
  if (p.a.refetch_threshold > 0.0f) {
    attn_full_kernel<DH><<<dim3(p.n_qt, p.a.H_kept, p.a.B), 256, FullCfg<DH>::kSmem, st>>>(p);
    SPT_TRY(launch_status());
  }
  return SPATTEN_OK;
}

}  // namespace

bool attn_tc_supported(const spatten_attn_args& a) {
  return a.quantized && a.q_dtype == SPATTEN_BF16 && (a.d_h == 64 || a.d_h == 128) && a.n_q > 1 &&
         a.n_q <= 256 * kMaxPairs;
}

int32_t attn_tc_launch(const AttnProblem& p, cudaStream_t st) {
  if (p.a.d_h == 64) return launch<64>(p, st);
  return launch<128>(p, st);
}

}  // namespace spt
