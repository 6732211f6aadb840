// K4: batched top-k selection with a deterministic tie-break and ascending-index output.
//
// SpAtten §IV.B "Top-k Engine" avoids a full sort: it finds the k-th largest value as a threshold
// with quick-select, filters the array against it and removes the gaps with a prefix-sum-driven
// zero eliminator.  The B200 form of the same three steps:
//   threshold  radix select over the order-preserving 32-bit image of each float: four 8-bit
//              digit passes, each a shared-memory histogram of the keys that still match the
//              known high digits; the CTAs of a thread-block cluster (one cluster per row) add
//              their histograms through distributed shared memory, so every CTA learns the
//              same digit without a trip through global memory.
//   filter     a key is kept if it is above the threshold T, or equal to T and among the first
//              (k - #above) equal keys in index order (ties go to the lower index).
//   eliminate  warp ballots + popc give each kept key its output slot (a block-wide exclusive
//              scan in index order), so the output is written in ascending index order.
// Each CTA keeps up to kResident keys of its chunk in shared memory; the rest (only for rows
// longer than clusters x kResident) is re-read from L2 in later passes.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace spt {
namespace {

constexpr int kTThreads = 512;
constexpr int kTWarps = kTThreads / 32;
constexpr int kResident = 48 * 1024;  // keys kept in shared memory per CTA (192 KB)

struct TArgs {
  const float* scores;
  int R, n;
  int64_t ld;
  int k;
  const int32_t* map;
  int64_t ld_map;
  int32_t* idx_out;
  int64_t ld_out;
  int32_t* comp_out;
  int32_t* status;
};

struct TShared {
  uint32_t hist[2][256];
  uint32_t red[256];
  uint32_t warp_a[kTWarps];
  uint32_t warp_b[kTWarps];
  uint32_t digit, above;
  uint32_t n_gt, n_eq;   // this CTA's counts after the last pass (read by peers)
  int nan_seen;
};

__device__ __forceinline__ uint32_t load_key(const TArgs& a, int r, int j, int* nan_seen) {
  const int64_t col = a.map ? a.map[static_cast<int64_t>(r) * a.ld_map + j] : j;
  const float f = a.scores[static_cast<int64_t>(r) * a.ld + col];
  if (f != f) *nan_seen = 1;
  return float_key(f);
}

__global__ void __launch_bounds__(kTThreads) topk_cluster_kernel(TArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int r = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) uint32_t keys_s[];
  __shared__ TShared sh;

  const int64_t out_base = static_cast<int64_t>(r) * a.ld_out;
  if (a.k == a.n) {  // everything is kept: positions 0..n-1
    for (int j = rank * kTThreads + tid; j < a.n; j += C * kTThreads) {
      a.idx_out[out_base + j] = j;
      if (a.comp_out) a.comp_out[out_base + j] = a.map[static_cast<int64_t>(r) * a.ld_map + j];
    }
    return;
  }
  if (a.k == 0) return;

  const int chunk = (a.n + C - 1) / C;
  const int c0 = min(a.n, rank * chunk), c1 = min(a.n, c0 + chunk);
  const int len = c1 - c0;
  const int resident = min(len, kResident);
  if (tid == 0) sh.nan_seen = 0;
  __syncthreads();
  int nan_local = 0;
  for (int j = tid; j < resident; j += kTThreads) keys_s[j] = load_key(a, r, c0 + j, &nan_local);
  if (nan_local) sh.nan_seen = 1;
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u;
  uint32_t krem = static_cast<uint32_t>(a.k);
  uint32_t above_local = 0u;  // keys of this chunk known to be above the final threshold
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* hist = sh.hist[pass & 1];
    if (tid < 256) hist[tid] = 0u;
    if (tid == 0) {
      sh.digit = 0u;
      sh.above = 0u;
    }
    __syncthreads();
    uint32_t above_pass = 0u;
    for (int base = 0; base < len; base += kTThreads) {
      const int j = base + tid;
      uint32_t bin = 256u;  // 256 = no histogram update
      if (j < len) {
        int dummy = 0;
        const uint32_t key = j < resident ? keys_s[j] : load_key(a, r, c0 + j, &dummy);
        const uint32_t hi = key & mask;
        if (hi == prefix)
          bin = (key >> shift) & 255u;
        else if (pass == 3 && hi > prefix)
          ++above_pass;
      }
      // warp-aggregated update: one shared atomic per distinct digit in the warp
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
    }
    if (pass == 3) {
      for (int o = 16; o > 0; o >>= 1) above_pass += __shfl_xor_sync(0xffffffffu, above_pass, o);
      if (lane == 0) sh.warp_a[warp] = above_pass;
    }
    cluster.sync();
    if (tid < 256) {
      uint32_t s = 0u;
      for (int c = 0; c < C; ++c) s += cluster.map_shared_rank(hist, c)[tid];
      sh.red[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending); find the digit holding rank krem
      uint32_t cnt[8];
      uint32_t tot = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = sh.red[255 - 8 * lane - i];
        tot += cnt[i];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - tot;
      const bool here = excl < krem && incl >= krem;
      const unsigned who = __ballot_sync(0xffffffffu, here);
      if (here && lane == static_cast<int>(__ffs(who) - 1)) {
        uint32_t run = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (run + cnt[i] >= krem) {
            sh.digit = static_cast<uint32_t>(255 - 8 * lane - i);
            sh.above = run;
            break;
          }
          run += cnt[i];
        }
      }
    }
    __syncthreads();
    const uint32_t d = sh.digit;
    if (pass == 3) {
      uint32_t gt = 0u;
      for (int w = 0; w < kTWarps; ++w) gt += sh.warp_a[w];
      for (uint32_t e = d + 1; e < 256u; ++e) gt += hist[e];
      above_local = gt;
      if (tid == 0) {
        sh.n_gt = gt;
        sh.n_eq = hist[d];
      }
    }
    krem -= sh.above;
    prefix |= d << shift;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix is now the threshold key T; krem keys equal to T are taken (lowest indices first)
  const uint32_t T = prefix;
  const uint32_t need_eq = krem;
  cluster.sync();  // every CTA's (n_gt, n_eq) is published
  uint32_t eq_before = 0u, sel_before = 0u;
  for (int c = 0; c < rank; ++c) {
    const TShared* peer = cluster.map_shared_rank(&sh, c);
    const uint32_t ne = peer->n_eq, ng = peer->n_gt;
    const uint32_t take = eq_before >= need_eq ? 0u : min(ne, need_eq - eq_before);
    sel_before += ng + take;
    eq_before += ne;
  }
  if (tid == 0 && sh.nan_seen) report(a.status, SPATTEN_E_NONFINITE);
  cluster.sync();  // peers' shared memory is no longer read after this point
  (void)above_local;

  // compaction in index order, kTThreads keys per tile
  uint32_t run_sel = sel_before, run_eq = eq_before;
  for (int base = 0; base < len; base += kTThreads) {
    const int j = base + tid;
    uint32_t key = 0u;
    if (j < len) {
      int dummy = 0;
      key = j < resident ? keys_s[j] : load_key(a, r, c0 + j, &dummy);
    }
    const bool gt = j < len && key > T;
    const bool eq = j < len && key == T;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) sh.warp_a[warp] = __popc(beq);
    __syncthreads();
    uint32_t eq_rank = run_eq + __popc(beq & ((1u << lane) - 1u));
    uint32_t eq_tile = 0u;
    for (int w = 0; w < kTWarps; ++w) {
      const uint32_t v = sh.warp_a[w];
      if (w < warp) eq_rank += v;
      eq_tile += v;
    }
    const bool sel = gt || (eq && eq_rank < need_eq);
    const unsigned bsel = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) sh.warp_b[warp] = __popc(bsel);
    __syncthreads();
    uint32_t pos = run_sel + __popc(bsel & ((1u << lane) - 1u));
    uint32_t sel_tile = 0u;
    for (int w = 0; w < kTWarps; ++w) {
      const uint32_t v = sh.warp_b[w];
      if (w < warp) pos += v;
      sel_tile += v;
    }
    if (sel && pos < static_cast<uint32_t>(a.k)) {
      a.idx_out[out_base + pos] = c0 + j;
      if (a.comp_out) a.comp_out[out_base + pos] = a.map[static_cast<int64_t>(r) * a.ld_map + c0 + j];
    }
    run_sel += sel_tile;
    run_eq += eq_tile;
    __syncthreads();
  }
}

int pick_cluster(int n) {
  // one CTA per 4096 keys, at most 8 (portable cluster size); 16 for very long rows when the
  // device can schedule such clusters
  int C = static_cast<int>(ceil_div(n, 4096));
  return std::max(1, std::min(C, 8));
}

}  // namespace

size_t topk_workspace_bytes(int R, int n, int k) {
  (void)R; (void)n; (void)k;
  return 0;
}

int32_t topk_launch(const TArgs& a, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    SPT_CUDA(cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kResident * 4));
    configured[dev] = true;
  }
  const int C = pick_cluster(a.n);
  const int chunk = static_cast<int>(ceil_div(a.n, C));
  const size_t smem = static_cast<size_t>(std::min(chunk, kResident)) * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, a.R, 1);
  cfg.blockDim = dim3(kTThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = C > 1 ? 1 : 0;   // a one-CTA row needs no cluster (implicit 1x1x1)
  SPT_CUDA(cudaLaunchKernelEx(&cfg, topk_cluster_kernel, a));
  return launch_status();
}

}  // namespace spt

extern "C" size_t spatten_topk_workspace_size(int32_t R, int32_t n, int32_t k) {
  return spt::topk_workspace_bytes(R, n, k);
}

extern "C" int32_t spatten_topk_select(const float* scores, int32_t R, int32_t n, int64_t ld,
                                       int32_t k, const int32_t* map, int64_t ld_map,
                                       int32_t* idx_out, int64_t ld_out, int32_t* comp_out,
                                       void* ws, size_t ws_bytes, int32_t* dev_status,
                                       void* stream) {
  using namespace spt;
  (void)ws;
  if (!scores || !idx_out) return SPATTEN_E_ARG;
  if (R < 1 || n < 1 || k < 0 || R > 65535) return SPATTEN_E_ARG;
  if (k > n) return SPATTEN_E_SHAPE;
  if (ld_out < k) return SPATTEN_E_SHAPE;
  if (!map && ld < n) return SPATTEN_E_SHAPE;
  if (map && ld_map < n) return SPATTEN_E_SHAPE;
  if (comp_out && !map) return SPATTEN_E_ARG;
  if (ws_bytes < topk_workspace_bytes(R, n, k)) return SPATTEN_E_WORKSPACE;
  TArgs a{scores, R, n, ld, k, map, ld_map, idx_out, ld_out, comp_out, dev_status};
  return topk_launch(a, as_stream(stream));
}
