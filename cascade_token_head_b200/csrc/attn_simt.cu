// K2f: attention with importance on CUDA cores (float32 arithmetic), any dtype, quantized or not.
//
// This is the path of the float32 configuration and the on-device cross-check of the
// tensor-core kernel.  Per CTA: one (sequence, kept head, 32-row query tile); keys stream through
// shared memory in 64-key tiles.  Three sweeps over the keys (SpAtten §IV.E):
//   A   MSB (or unquantized) pass: online row max / exp-sum  ->  refetch flag = 1/ell < theta
//   A'  only if some row of the tile is flagged: the same stats with the full 12-bit K for the
//       flagged rows (the LSB plane is read only then: "fetches LSBs only when ... flat")
//   B   final probabilities P = exp(S - m)/ell, column sums of P (token importance), O = P V
// Column sums are reduced in a fixed order (lanes own keys, warps summed in warp order), then
// written as this CTA's partial; attn_reduce adds the partials in a fixed order.
#include "attention.cuh"

namespace spt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = kSimtRows;          // 32 query rows per CTA, 4 per warp
constexpr int kRowsPerWarp = kRows / kWarps;
constexpr int kKeys = 64;                 // keys per tile, 2 per lane

template <int DH>
struct SimtSmem {
  float q[kRows][DH];
  float k_hi[kKeys][DH + 1];   // MSB part (or unquantized K)
  float k_lo[kKeys][DH + 1];   // LSB part  scale * LSB
  float v_hi[kKeys][DH + 1];
  float v_lo[kKeys][DH + 1];
  float p[kWarps][kKeys];
  float col[kWarps][kKeys];
  float hsum[kWarps];
};

template <typename T>
__device__ __forceinline__ float ldf(const void* base, int64_t off) {
  return ld_as_float(static_cast<const T*>(base) + off);
}

// load one key tile (rows j0 .. j0+kKeys-1) of K or V into shared memory (hi and optionally lo)
// keep (V under local value pruning): key j is loaded iff keep[j] != 0; dropped keys read as 0
template <int DH, typename KVT>
__device__ void load_tile(const spatten_attn_args& a, int b, int h, int j0, bool is_v, bool want_lo,
                          float (*hi)[DH + 1], float (*lo)[DH + 1], const uint8_t* keep) {
  if (!is_v) keep = nullptr;
  if (a.quantized) {
    const int8_t* msb = is_v ? a.v_msb : a.k_msb;
    const uint8_t* lsb = is_v ? a.v_lsb : a.k_lsb;
    const float s = (is_v ? a.v_scale : a.k_scale)[b * a.H + h];
    for (int e = threadIdx.x; e < kKeys * DH; e += kThreads) {
      const int jj = e / DH, d = e % DH, j = j0 + jj;
      float vh = 0.0f, vl = 0.0f;
      if (j < a.n_kv && (!keep || keep[j])) {
        const int64_t row = a.kv_idx ? a.kv_idx[static_cast<int64_t>(b) * a.kv_idx_ld + j] : j;
        const int64_t base = (static_cast<int64_t>(b) * a.H + h) * a.kv_cap + row;
        vh = s * 16.0f * static_cast<float>(msb[base * DH + d]);
        if (want_lo) {
          const uint8_t byte = lsb[base * (DH / 2) + d / 2];
          vl = s * static_cast<float>((d & 1) ? (byte >> 4) : (byte & 15));
        }
      }
      hi[jj][d] = vh;
      if (want_lo) lo[jj][d] = vl;
    }
  } else {
    const void* src = is_v ? a.v : a.k;
    for (int e = threadIdx.x; e < kKeys * DH; e += kThreads) {
      const int jj = e / DH, d = e % DH, j = j0 + jj;
      float v = 0.0f;
      if (j < a.n_kv && (!keep || keep[j])) v = ldf<KVT>(src, (static_cast<int64_t>(b) * a.n_kv + j) * a.kv_ld_tok + static_cast<int64_t>(h) * DH + d);
      hi[jj][d] = v;
    }
  }
}

template <int DH, typename QT, typename KVT>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnProblem p) {
  const spatten_attn_args& a = p.a;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<DH>& sm = *reinterpret_cast<SimtSmem<DH>*>(smem_raw);
  const int qt = blockIdx.x, slot = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = qt * kRows;
  const int h = head_of_slot(a, b, slot);
  QT* o = static_cast<QT*>(a.o);

  if (slot >= a.H_kept) {  // pruned head: zero its output block
    if (h < 0) return;
    for (int e = threadIdx.x; e < kRows * DH; e += kThreads) {
      const int i = i0 + e / DH, d = e % DH;
      if (i < a.n_q) st_from_float(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok + static_cast<int64_t>(h) * DH + d, 0.0f);
    }
    return;
  }

  const QT* q = static_cast<const QT*>(a.q);
  for (int e = threadIdx.x; e < kRows * DH; e += kThreads) {
    const int r = e / DH, d = e % DH, i = i0 + r;
    sm.q[r][d] = i < a.n_q ? ld_as_float(q + (static_cast<int64_t>(b) * a.n_q + i) * a.q_ld_tok + static_cast<int64_t>(h) * DH + d) : 0.0f;
  }

  const float scale = a.sm_scale;
  float m[kRowsPerWarp], l[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) { m[r] = -INFINITY; l[r] = 0.0f; }

  const int n_tiles = (a.n_kv + kKeys - 1) / kKeys;
  // ---- pass A: MSB / unquantized statistics --------------------------------------------------
  for (int t = 0; t < n_tiles; ++t) {
    __syncthreads();
    load_tile<DH, KVT>(a, b, h, t * kKeys, false, false, sm.k_hi, sm.k_lo, nullptr);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int ri = warp * kRowsPerWarp + r;
      float s[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int jj = lane + 32 * c;
        float acc = 0.0f;
#pragma unroll 16
        for (int d = 0; d < DH; ++d) acc = fmaf(sm.q[ri][d], sm.k_hi[jj][d], acc);
        s[c] = (t * kKeys + jj < a.n_kv) ? acc * scale : -INFINITY;
      }
      const float tmax = warp_max(fmaxf(s[0], s[1]));
      const float mn = fmaxf(m[r], tmax);
      const float add = warp_sum(expf(s[0] - mn) + expf(s[1] - mn));
      l[r] = (m[r] == -INFINITY ? 0.0f : l[r] * expf(m[r] - mn)) + add;
      m[r] = mn;
    }
  }
  bool flag[kRowsPerWarp];
  bool mine = false;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int i = i0 + warp * kRowsPerWarp + r;
    flag[r] = a.quantized && i < a.n_q && (1.0f / l[r] < a.refetch_threshold);
    mine |= flag[r];
  }
  const bool any_flag = __syncthreads_or(mine) != 0;

  // ---- pass A': full-precision statistics of the flagged rows ---------------------------------
  if (any_flag) {
    float mf[kRowsPerWarp], lf[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) { mf[r] = -INFINITY; lf[r] = 0.0f; }
    for (int t = 0; t < n_tiles; ++t) {
      __syncthreads();
      load_tile<DH, KVT>(a, b, h, t * kKeys, false, true, sm.k_hi, sm.k_lo, nullptr);
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        if (!flag[r]) continue;   // warp-uniform
        const int ri = warp * kRowsPerWarp + r;
        float s[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int jj = lane + 32 * c;
          float acc = 0.0f;
#pragma unroll 16
          for (int d = 0; d < DH; ++d) acc = fmaf(sm.q[ri][d], sm.k_hi[jj][d] + sm.k_lo[jj][d], acc);
          s[c] = (t * kKeys + jj < a.n_kv) ? acc * scale : -INFINITY;
        }
        const float tmax = warp_max(fmaxf(s[0], s[1]));
        const float mn = fmaxf(mf[r], tmax);
        const float add = warp_sum(expf(s[0] - mn) + expf(s[1] - mn));
        lf[r] = (mf[r] == -INFINITY ? 0.0f : lf[r] * expf(mf[r] - mn)) + add;
        mf[r] = mn;
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
      if (flag[r]) { m[r] = mf[r]; l[r] = lf[r]; }
  }

  // ---- pass B: probabilities, column sums, outputs --------------------------------------------
  constexpr int DPL = DH / 32;   // output dims per lane
  float acc_o[kRowsPerWarp][DPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int c = 0; c < DPL; ++c) acc_o[r][c] = 0.0f;
  float inv_l[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) inv_l[r] = 1.0f / l[r];

  const int64_t part_row = ((static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt) * a.n_kv;
  const uint8_t* vkeep = p.v_mask ? p.v_mask + (static_cast<int64_t>(b) * a.H_kept + slot) * a.n_kv : nullptr;
  for (int t = 0; t < n_tiles; ++t) {
    __syncthreads();
    load_tile<DH, KVT>(a, b, h, t * kKeys, false, any_flag, sm.k_hi, sm.k_lo, nullptr);
    load_tile<DH, KVT>(a, b, h, t * kKeys, true, any_flag, sm.v_hi, sm.v_lo, vkeep);
    __syncthreads();
    float col[2] = {0.0f, 0.0f};
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int ri = warp * kRowsPerWarp + r;
      const bool valid_row = i0 + ri < a.n_q;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int jj = lane + 32 * c;
        float acc = 0.0f;
        if (flag[r]) {
#pragma unroll 16
          for (int d = 0; d < DH; ++d) acc = fmaf(sm.q[ri][d], sm.k_hi[jj][d] + sm.k_lo[jj][d], acc);
        } else {
#pragma unroll 16
          for (int d = 0; d < DH; ++d) acc = fmaf(sm.q[ri][d], sm.k_hi[jj][d], acc);
        }
        float pr = 0.0f;
        if (valid_row && t * kKeys + jj < a.n_kv) pr = expf(acc * scale - m[r]) * inv_l[r];
        sm.p[warp][jj] = pr;
        col[c] += pr;
      }
      __syncwarp();
#pragma unroll
      for (int c = 0; c < DPL; ++c) {
        const int d = lane + 32 * c;
        float o_acc = acc_o[r][c];
        if (flag[r]) {
          for (int jj = 0; jj < kKeys; ++jj) o_acc = fmaf(sm.p[warp][jj], sm.v_hi[jj][d] + sm.v_lo[jj][d], o_acc);
        } else {
          for (int jj = 0; jj < kKeys; ++jj) o_acc = fmaf(sm.p[warp][jj], sm.v_hi[jj][d], o_acc);
        }
        acc_o[r][c] = o_acc;
      }
      __syncwarp();
    }
    sm.col[warp][lane] = col[0];
    sm.col[warp][lane + 32] = col[1];
    __syncthreads();
    if (threadIdx.x < kKeys) {
      const int j = t * kKeys + threadIdx.x;
      float s = 0.0f;
      for (int w = 0; w < kWarps; ++w) s += sm.col[w][threadIdx.x];
      if (j < a.n_kv) p.tok_part[part_row + j] = s;
    }
  }

  // ---- epilogue: O, head importance, flags ------------------------------------------------------
  float habs = 0.0f;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int i = i0 + warp * kRowsPerWarp + r;
    if (i >= a.n_q) continue;
#pragma unroll
    for (int c = 0; c < DPL; ++c) {
      const int d = lane + 32 * c;
      habs += fabsf(acc_o[r][c]);
      st_from_float(o + (static_cast<int64_t>(b) * a.n_q + i) * a.o_ld_tok + static_cast<int64_t>(h) * DH + d, acc_o[r][c]);
    }
    if (lane == 0 && a.refetch_flags)
      a.refetch_flags[(static_cast<int64_t>(b) * a.H + h) * a.refetch_flags_ld + i] = flag[r] ? 1 : 0;
  }
  habs = warp_sum(habs);
  int nflag = 0;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) nflag += flag[r] ? 1 : 0;
  if (lane == 0) sm.hsum[warp] = habs;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.0f;
    for (int w = 0; w < kWarps; ++w) s += sm.hsum[w];
    p.head_part[(static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt] = s;
  }
  if (lane == 0 && nflag && a.refetch_count) atomicAdd(a.refetch_count, nflag);
}

template <int DH, typename QT, typename KVT>
int32_t launch_simt(const AttnProblem& p, cudaStream_t st) {
  const spatten_attn_args& a = p.a;
  const size_t smem = sizeof(SimtSmem<DH>);
  static DeviceOnce once;
  int dev = 0;
  SPT_TRY(once_per_device(once, &dev, [smem](int) -> int32_t {
    SPT_CUDA(cudaFuncSetAttribute(attn_simt_kernel<DH, QT, KVT>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
    return SPATTEN_OK;
  }));
  const int slots = a.H_kept + (a.zero_pruned_heads ? a.H - a.H_kept : 0);
  dim3 grid(p.n_qt, slots, a.B);
  attn_simt_kernel<DH, QT, KVT><<<grid, kThreads, smem, st>>>(p);
  return launch_status();
}

template <int DH>
int32_t dispatch_types(const AttnProblem& p, cudaStream_t st) {
  const spatten_attn_args& a = p.a;
  const bool qb = a.q_dtype == SPATTEN_BF16;
  const bool kvb = a.quantized ? qb : a.kv_dtype == SPATTEN_BF16;
  if (qb && kvb) return launch_simt<DH, __nv_bfloat16, __nv_bfloat16>(p, st);
  if (qb) return launch_simt<DH, __nv_bfloat16, float>(p, st);
  if (kvb) return launch_simt<DH, float, __nv_bfloat16>(p, st);
  return launch_simt<DH, float, float>(p, st);
}

}  // namespace

int32_t attn_simt_launch(const AttnProblem& p, cudaStream_t st) {
  if (p.a.d_h == 64) return dispatch_types<64>(p, st);
  if (p.a.d_h == 128) return dispatch_types<128>(p, st);
  return SPATTEN_E_UNSUPPORTED;
}


}  // namespace spt
