// Fixed-order reduction of the attention kernels' per-CTA partial sums into the cumulative token
// importance (SpAtten §II "Cascade pruning": the column sums of P accumulate over heads, queries
// and layers) and head importance (sum |O|).
//
// A CTA takes 64 keys of one sequence; its 256 threads form 4 groups of 64, group g summing, for
// its key, the partial rows of the kept heads slot = g, g+4, g+8, ... (each head's 128-row query
// tiles, then its packed refetch tiles) in that order; the 4 group sums are then added in group
// order.  Every key is summed in the same order on every run, so results are bit-identical.
// For local value pruning the same partials also give each head's own column sums.
#include "attention.cuh"

namespace spt {
namespace {

constexpr int kKeysPerCta = 64;
constexpr int kGroups = 4;

__device__ __forceinline__ int refetch_rows(const AttnProblem& p, int b, int slot) {
  if (!p.flag_cnt) return 0;
  int total = 0;
  const int32_t* c = p.flag_cnt + (static_cast<int64_t>(b) * p.a.H_kept + slot) * p.n_pair;
  for (int pp = 0; pp < p.n_pair; ++pp) total += c[pp];
  return total;
}

__global__ void __launch_bounds__(256) attn_reduce_kernel(AttnProblem p) {
  const spatten_attn_args& a = p.a;
  const int b = blockIdx.y;
  extern __shared__ int nfull_s[];   // [H_kept] packed refetch tiles per kept head
  __shared__ float grp[kGroups][kKeysPerCta];
  for (int slot = threadIdx.x; slot < a.H_kept; slot += blockDim.x)
    nfull_s[slot] = (refetch_rows(p, b, slot) + 127) / 128;
  __syncthreads();

  const int nblk_tok = (a.n_kv + kKeysPerCta - 1) / kKeysPerCta;
  if (static_cast<int>(blockIdx.x) < nblk_tok) {
    if (!a.tok_imp) return;
    const int kk = threadIdx.x % kKeysPerCta, g = threadIdx.x / kKeysPerCta;
    const int j = blockIdx.x * kKeysPerCta + kk;
    float s = 0.0f;
    if (j < a.n_kv) {
      for (int slot = g; slot < a.H_kept; slot += kGroups) {
        const float* row = p.tok_part + (static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt * a.n_kv + j;
        float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        int qt = 0;
        for (; qt + 4 <= p.n_qt; qt += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) s4[u] += row[static_cast<int64_t>(qt + u) * a.n_kv];
        }
        for (; qt < p.n_qt; ++qt) s4[0] += row[static_cast<int64_t>(qt) * a.n_kv];
        s += (s4[0] + s4[1]) + (s4[2] + s4[3]);
        const int nf = nfull_s[slot];
        const float* frow = p.full_part ? p.full_part + (static_cast<int64_t>(b) * a.H_kept + slot) * 2 * p.n_pair * a.n_kv + j
                                        : nullptr;
        for (int u = 0; u < nf; ++u) s += frow[static_cast<int64_t>(u) * a.n_kv];
      }
    }
    grp[g][kk] = s;
    __syncthreads();
    if (g == 0 && j < a.n_kv) {
      const float t = ((grp[0][kk] + grp[1][kk]) + grp[2][kk]) + grp[3][kk];
      const int64_t dst = a.tok_imp_map ? a.tok_imp_map[static_cast<int64_t>(b) * a.tok_imp_map_ld + j] : j;
      a.tok_imp[static_cast<int64_t>(b) * a.tok_imp_ld + dst] += t;
    }
  } else {
    if (!a.head_imp) return;
    for (int slot = threadIdx.x; slot < a.H_kept; slot += blockDim.x) {
      float s = 0.0f;
      for (int qt = 0; qt < p.n_qt; ++qt) s += p.head_part[(static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt + qt];
      for (int u = 0; u < nfull_s[slot]; ++u) s += p.full_head[(static_cast<int64_t>(b) * a.H_kept + slot) * 2 * p.n_pair + u];
      const int h = a.head_idx ? a.head_idx[static_cast<int64_t>(b) * a.head_idx_ld + slot] : slot;
      a.head_imp[static_cast<int64_t>(b) * a.H + h] += s;
    }
  }
}

// Local value pruning: the column sums of each kept head's probabilities, head_col[b][slot][j],
// from the same partials and in the same order as one head's share of the token reduction.
__global__ void __launch_bounds__(256) attn_head_colsum_kernel(AttnProblem p) {
  const spatten_attn_args& a = p.a;
  const int slot = blockIdx.y, b = blockIdx.z;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= a.n_kv) return;
  const float* row = p.tok_part + (static_cast<int64_t>(b) * a.H_kept + slot) * p.n_qt * a.n_kv + j;
  float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  int qt = 0;
  for (; qt + 4 <= p.n_qt; qt += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) s4[u] += row[static_cast<int64_t>(qt + u) * a.n_kv];
  }
  for (; qt < p.n_qt; ++qt) s4[0] += row[static_cast<int64_t>(qt) * a.n_kv];
  float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  if (p.full_part) {
    const int nf = (refetch_rows(p, b, slot) + 127) / 128;
    const float* frow = p.full_part + (static_cast<int64_t>(b) * a.H_kept + slot) * 2 * p.n_pair * a.n_kv + j;
    for (int u = 0; u < nf; ++u) s += frow[static_cast<int64_t>(u) * a.n_kv];
  }
  p.head_col[(static_cast<int64_t>(b) * a.H_kept + slot) * a.n_kv + j] = s;
}

// V mask of the second run: 1 for the v_keep kept keys of each (sequence, kept head), else 0
__global__ void __launch_bounds__(256) attn_value_mask_kernel(AttnProblem p, uint8_t* mask) {
  const spatten_attn_args& a = p.a;
  const int64_t row = blockIdx.y;   // b * H_kept + slot
  uint8_t* m = mask + row * a.n_kv;
  for (int j = threadIdx.x; j < a.n_kv; j += blockDim.x) m[j] = 0;
  __syncthreads();
  const int32_t* sel = p.v_sel + row * a.v_keep;
  for (int c = threadIdx.x; c < a.v_keep; c += blockDim.x) m[sel[c]] = 1;
}

}  // namespace

int32_t attn_head_colsum_launch(const AttnProblem& p, cudaStream_t st) {
  attn_head_colsum_kernel<<<dim3(static_cast<unsigned>(ceil_div(p.a.n_kv, 256)), p.a.H_kept, p.a.B), 256, 0, st>>>(p);
  return launch_status();
}

int32_t attn_value_mask_launch(const AttnProblem& p, uint8_t* mask, cudaStream_t st) {
  attn_value_mask_kernel<<<dim3(1, p.a.B * p.a.H_kept), 256, 0, st>>>(p, mask);
  return launch_status();
}

int32_t attn_reduce_launch(const AttnProblem& p, cudaStream_t st) {
  const int nblk = (p.a.n_kv + kKeysPerCta - 1) / kKeysPerCta + 1;
  attn_reduce_kernel<<<dim3(nblk, p.a.B), 256, sizeof(int) * p.a.H_kept, st>>>(p);
  return launch_status();
}

}  // namespace spt
