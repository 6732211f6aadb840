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
// longer than clusters x kResident) is streamed again from L2 in every pass, eight keys per
// thread with 16-byte loads, and compacted with block-wide prefix sums of per-thread counts.
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
  const int32_t* only_rows = nullptr;   // device [R] or NULL: rows with 0 are skipped (fallback use)
};

struct TShared {
  uint32_t hist[2][256];
  uint32_t red[256];
  uint32_t warp_a[kTWarps];
  uint32_t warp_b[kTWarps];
  uint32_t scan[2][kTWarps];
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

// 8 consecutive keys of row r starting at column j (absolute), columns >= lim invalid; two 16-byte
// loads when the row is read directly and aligned, otherwise element loads
__device__ __forceinline__ void load8_keys(const TArgs& a, int r, int j, int lim, bool vec, uint32_t* key, bool* ok,
                                           int* nan_seen) {
  if (vec && j + 7 < lim) {
    const float4* p = reinterpret_cast<const float4*>(a.scores + static_cast<int64_t>(r) * a.ld + j);
    const float4 f0 = __ldg(p), f1 = __ldg(p + 1);
    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (f[u] != f[u]) *nan_seen = 1;
      key[u] = float_key(f[u]);
      ok[u] = true;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      ok[u] = j + u < lim;
      key[u] = ok[u] ? load_key(a, r, j + u, nan_seen) : 0u;
    }
  }
}

// exclusive prefix sum of one value per thread over the block (all threads must call); wt is a
// [kTWarps] scratch array that must not be reused before every thread has passed the next block
// barrier (callers alternate two arrays)
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wt, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) wt[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < kTWarps ? wt[lane] : 0u;
#pragma unroll
    for (int o = 1; o < kTWarps; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += t;
    }
    if (lane < kTWarps) wt[lane] = x;   // inclusive warp prefixes
  }
  __syncthreads();
  total = wt[kTWarps - 1];
  return (warp > 0 ? wt[warp - 1] : 0u) + inc - v;
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
  if (a.only_rows && !a.only_rows[r]) return;   // uniform over the cluster: no barrier skipped
  if (a.k == a.n) {  // everything is kept: positions 0..n-1
    for (int j = rank * kTThreads + tid; j < a.n; j += C * kTThreads) {
      if (a.idx_out) a.idx_out[out_base + j] = j;
      if (a.comp_out) a.comp_out[out_base + j] = a.map[static_cast<int64_t>(r) * a.ld_map + j];
    }
    return;
  }
  if (a.k == 0) return;

  // chunks start on a multiple of 4 keys so that direct rows can be read with 16-byte loads
  const int chunk = (((a.n + C - 1) / C) + 3) & ~3;
  const int c0 = min(a.n, rank * chunk), c1 = min(a.n, c0 + chunk);
  const int len = c1 - c0;
  const int resident = min(len, kResident);
  const bool vec = a.map == nullptr && (a.ld & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
  if (tid == 0) sh.nan_seen = 0;
  __syncthreads();
  int nan_local = 0;
  // resident part: 8 keys per thread per step, 16-byte loads when possible
  for (int base = 0; base < resident; base += 8 * kTThreads) {
    const int j = base + 8 * tid;
    uint32_t key[8];
    bool ok[8];
    load8_keys(a, r, c0 + j, c0 + resident, vec, key, ok, &nan_local);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (ok[u]) keys_s[j + u] = key[u];
  }
  if (nan_local) sh.nan_seen = 1;
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u;
  uint32_t krem = static_cast<uint32_t>(a.k);
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
    auto count_key = [&](uint32_t key, bool ok) {
      uint32_t bin = 256u;  // 256 = no histogram update
      if (ok) {
        const uint32_t hi = key & mask;
        if (hi == prefix)
          bin = (key >> shift) & 255u;
        else if (pass == 3 && hi > prefix)
          ++above_pass;
      }
      // warp-aggregated update: one shared atomic per distinct digit in the warp; after the first
      // pass most warps hold no key that still matches the prefix and skip it
      if (pass == 0 || __any_sync(0xffffffffu, bin < 256u)) {
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
      }
    };
    for (int base = 0; base < resident; base += 4 * kTThreads) {   // four keys per thread (16-byte reads)
      const int j = base + 4 * tid;
      uint4 k4 = make_uint4(0u, 0u, 0u, 0u);
      if (j + 3 < resident) {
        k4 = *reinterpret_cast<const uint4*>(keys_s + j);
      } else {
        if (j < resident) k4.x = keys_s[j];
        if (j + 1 < resident) k4.y = keys_s[j + 1];
        if (j + 2 < resident) k4.z = keys_s[j + 2];
      }
      count_key(k4.x, j < resident);
      count_key(k4.y, j + 1 < resident);
      count_key(k4.z, j + 2 < resident);
      count_key(k4.w, j + 3 < resident);
    }
    for (int base = resident; base < len; base += 8 * kTThreads) {   // streamed part (long rows)
      uint32_t key[8];
      bool ok[8];
      int dummy = 0;
      load8_keys(a, r, c0 + base + 8 * tid, c0 + len, vec, key, ok, &dummy);
#pragma unroll
      for (int u = 0; u < 8; ++u) count_key(key[u], ok[u]);
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
    if (pass == 3 && tid == 0) {
      uint32_t gt = 0u;
      for (int w = 0; w < kTWarps; ++w) gt += sh.warp_a[w];
      for (uint32_t e = d + 1; e < 256u; ++e) gt += hist[e];
      sh.n_gt = gt;
      sh.n_eq = hist[d];
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

  // compaction in index order, eight consecutive keys per thread per tile: one block scan of the
  // packed per-thread counts (above T in the low half, equal to T in the high half) places every
  // thread's keys; equal keys are taken in index order while the row still needs them
  uint32_t run_sel = sel_before, run_eq = eq_before;
  int tile = 0;
  auto compact8 = [&](int j, const uint32_t* key, const bool* ok) {
    uint32_t gtc = 0u, eqc = 0u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      gtc += (ok[u] && key[u] > T) ? 1u : 0u;
      eqc += (ok[u] && key[u] == T) ? 1u : 0u;
    }
    uint32_t tot;
    const uint32_t pre = block_excl_scan(gtc | (eqc << 16), sh.scan[tile & 1], tot);
    ++tile;
    const uint32_t rem = need_eq > run_eq ? need_eq - run_eq : 0u;   // equal keys still wanted
    const uint32_t pre_eq = pre >> 16;
    uint32_t pos = run_sel + (pre & 0xFFFFu) + min(pre_eq, rem);
    uint32_t er = run_eq + pre_eq;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool gt = ok[u] && key[u] > T;
      const bool eq = ok[u] && key[u] == T;
      const bool sel = gt || (eq && er < need_eq);
      er += eq ? 1u : 0u;
      if (sel) {
        if (pos < static_cast<uint32_t>(a.k)) {
          if (a.idx_out) a.idx_out[out_base + pos] = c0 + j + u;
          if (a.comp_out) a.comp_out[out_base + pos] = a.map[static_cast<int64_t>(r) * a.ld_map + c0 + j + u];
        }
        ++pos;
      }
    }
    run_sel += (tot & 0xFFFFu) + min(tot >> 16, rem);
    run_eq += tot >> 16;
  };
  for (int base = 0; base < resident; base += 8 * kTThreads) {
    const int j = base + 8 * tid;
    uint32_t key[8];
    bool ok[8];
    if (j + 7 < resident) {
      const uint4 k0 = *reinterpret_cast<const uint4*>(keys_s + j);
      const uint4 k1 = *reinterpret_cast<const uint4*>(keys_s + j + 4);
      key[0] = k0.x; key[1] = k0.y; key[2] = k0.z; key[3] = k0.w;
      key[4] = k1.x; key[5] = k1.y; key[6] = k1.z; key[7] = k1.w;
#pragma unroll
      for (int u = 0; u < 8; ++u) ok[u] = true;
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        ok[u] = j + u < resident;
        key[u] = ok[u] ? keys_s[j + u] : 0u;
      }
    }
    compact8(j, key, ok);
  }
  for (int base = resident; base < len; base += 8 * kTThreads) {   // streamed keys
    const int j = base + 8 * tid;
    uint32_t key[8];
    bool ok[8];
    int dummy = 0;
    load8_keys(a, r, c0 + j, c0 + len, vec, key, ok, &dummy);
    compact8(j, key, ok);
  }
}

// ------------------------------------------------------------------------------------------------
// Short rows (n <= 8192): the row's keys live in registers, sixteen consecutive keys per thread, one
// warp per row (n <= 512, four rows per CTA, no block barrier) or one CTA of G warps per row (G = 4
// up to 2048 keys, 16 up to 8192).  The
// threshold T (the k-th largest key) is found digit by digit, two bits per round: of the candidates
// T | j << b (j = 1..3) the largest one with at least k keys at or above it is kept, so after 16
// rounds T is the largest value with count(key >= T) >= k.  Counting is a compare per key and an
// integer warp reduction (__reduce_add_sync); no histogram, no atomics.  need_eq = k - count(key > T)
// keys equal to T are taken in index order; one packed scan places every thread's selected keys.
// ------------------------------------------------------------------------------------------------
constexpr int kSKeys = 16;

template <int G>
__global__ void __launch_bounds__(G == 1 ? 128 : 32 * G) topk_small_kernel(TArgs a) {
  constexpr int RPC = G == 1 ? 4 : 1;   // rows per CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * RPC + (G == 1 ? warp : 0);
  const int t = G == 1 ? lane : static_cast<int>(threadIdx.x);   // thread within the row
  __shared__ uint32_t red[2][2][G];    // [round parity][word][warp]
  __shared__ uint32_t wscan[G];
  __shared__ int nan_any;
  if (r >= a.R) return;                // G == 1: the whole warp; G > 1: never (grid = R)
  const int64_t out_base = static_cast<int64_t>(r) * a.ld_out;
  if (a.k == 0) return;
  if (a.k == a.n) {
    for (int j = t; j < a.n; j += 32 * G) {
      if (a.idx_out) a.idx_out[out_base + j] = j;
      if (a.comp_out) a.comp_out[out_base + j] = a.map[static_cast<int64_t>(r) * a.ld_map + j];
    }
    return;
  }
  if (G > 1 && threadIdx.x == 0) nan_any = 0;

  // keys t*16 .. t*16+15 of the row; missing keys are 0 (below every candidate, which is >= 1)
  uint32_t key[kSKeys];
  int nan_local = 0;
  const int j0 = t * kSKeys;
  const bool vec = a.map == nullptr && (a.ld & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
  if (vec && j0 + kSKeys <= a.n) {
    const float4* p = reinterpret_cast<const float4*>(a.scores + static_cast<int64_t>(r) * a.ld + j0);
#pragma unroll
    for (int q = 0; q < kSKeys / 4; ++q) {
      const float4 f = __ldg(p + q);
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        nan_local |= fv[u] != fv[u];
        key[4 * q + u] = float_key(fv[u]);
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < kSKeys; ++u) key[u] = j0 + u < a.n ? load_key(a, r, j0 + u, &nan_local) : 0u;
  }
  int round = 0;
  // counts of keys >= c1, c2, c3 over the row: (c1 | c2 << 16) and c3
  auto count3 = [&](uint32_t c1, uint32_t c2, uint32_t c3, uint32_t& n1, uint32_t& n2, uint32_t& n3) {
    uint32_t x = 0u, y = 0u;
#pragma unroll
    for (int u = 0; u < kSKeys; ++u) {
      x += (key[u] >= c1 ? 1u : 0u) + (key[u] >= c2 ? 0x10000u : 0u);
      y += key[u] >= c3 ? 1u : 0u;
    }
    x = __reduce_add_sync(0xffffffffu, x);
    y = __reduce_add_sync(0xffffffffu, y);
    if (G > 1) {
      const int pr = round & 1;
      if (lane == 0) {
        red[pr][0][warp] = x;
        red[pr][1][warp] = y;
      }
      __syncthreads();
      x = 0u;
      y = 0u;
#pragma unroll
      for (int w = 0; w < G; ++w) {
        x += red[pr][0][w];
        y += red[pr][1][w];
      }
    }
    ++round;
    n1 = x & 0xFFFFu;
    n2 = x >> 16;
    n3 = y;
  };
  const uint32_t k = static_cast<uint32_t>(a.k);
  uint32_t T = 0u;
#pragma unroll 1
  for (int b = 30; b >= 0; b -= 2) {
    uint32_t n1, n2, n3;
    count3(T | (1u << b), T | (2u << b), T | (3u << b), n1, n2, n3);
    T |= static_cast<uint32_t>((n1 >= k) + (n2 >= k) + (n3 >= k)) << b;
  }
  uint32_t n_gt, d1, d2;
  if (T == 0xFFFFFFFFu) {
    n_gt = 0u;
  } else {
    count3(T + 1u, 0xFFFFFFFFu, 0xFFFFFFFFu, n_gt, d1, d2);
  }
  const uint32_t need_eq = k - n_gt;
  if (G > 1) {
    if (nan_local) nan_any = 1;
    __syncthreads();
    nan_local = nan_any;
  } else {
    nan_local = __any_sync(0xffffffffu, nan_local);
  }
  if (nan_local && t == 0) report(a.status, SPATTEN_E_NONFINITE);

  // ordered compaction: exclusive scan of packed (above T | equal to T << 16) per-thread counts
  uint32_t gtc = 0u, eqc = 0u;
#pragma unroll
  for (int u = 0; u < kSKeys; ++u) {
    gtc += key[u] > T ? 1u : 0u;
    eqc += (j0 + u < a.n && key[u] == T) ? 1u : 0u;
  }
  const uint32_t v = gtc | (eqc << 16);
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  uint32_t pre = inc - v;
  if (G > 1) {
    if (lane == 31) wscan[warp] = inc;
    __syncthreads();
    uint32_t before = 0u;
    for (int w = 0; w < warp; ++w) before += wscan[w];
    pre += before;
  }
  uint32_t pos = (pre & 0xFFFFu) + min(pre >> 16, need_eq);
  uint32_t er = pre >> 16;
#pragma unroll
  for (int u = 0; u < kSKeys; ++u) {
    const bool gt = key[u] > T;
    const bool eq = j0 + u < a.n && key[u] == T;
    const bool sel = gt || (eq && er < need_eq);
    er += eq ? 1u : 0u;
    if (sel) {
      if (pos < k) {
        if (a.idx_out) a.idx_out[out_base + pos] = j0 + u;
        if (a.comp_out) a.comp_out[out_base + pos] = a.map[static_cast<int64_t>(r) * a.ld_map + j0 + u];
      }
      ++pos;
    }
  }
}

// ------------------------------------------------------------------------------------------------
// Long rows (n >= kStreamMin, scores read directly, caller workspace given): two streaming passes.
//  sample   one CTA per row sorts 16 K keys (64 evenly spaced runs of 256) and takes, around the
//           sample rank of the k-th key (+-4 sigma of the sampling error + 16), a bracket
//           [e64, e0] cut into 64 sub-bins at sample quantiles e0 >= e1 >= ... >= e64
//  filter   per chunk of 16 K keys: the count above e0, a histogram of the bracket's keys over the
//           sub-bins, and the bracket's keys (key, index) appended to the row's candidate buffer
//  resolve  one CTA per row: the sub-bin holding the k-th key, the exact threshold among that
//           sub-bin's candidates as the (need)-th largest of (key, ~index) (ties to the lower
//           index), and every chunk's output offset
//  output   per chunk: key > T, or key = T and index <= T_index, written in index order
// A row whose k-th key fell outside the bracket, or whose buffers overflowed, is marked and done
// again by the cluster kernel (only_rows).
// ------------------------------------------------------------------------------------------------
constexpr int kStreamMin = 65536;
constexpr int kSRuns = 64, kSRun = 256, kSamples = kSRuns * kSRun;   // 16 K sample keys per row
constexpr int kBins = 64;
constexpr int kChunk = 16384;                                           // keys per filter/output CTA
constexpr int kCThreads2 = 512;                                         // threads of filter/output
constexpr int kBinCap = 8192;                                           // candidates of one sub-bin

struct StreamWs {
  uint32_t* edges;      // [R][kBins + 1]
  uint32_t* hist;       // [R][kBins]           (zeroed per call)
  uint32_t* ccount;     // [R]                   (zeroed per call)
  uint32_t* chunk_gt;   // [R][nchunk]
  uint2* cand;          // [R][cap]  (key, index)
  uint32_t* chunk_off;  // [R][nchunk]
  uint32_t* res;        // [R][4]   valid, T key, T index
  int32_t* fallback;    // [R]
  int cap, nchunk;
};

__device__ __forceinline__ int bin_of(uint32_t key, const uint32_t* e) {
  // number of edges e1..e63 at or above key (edges descending): bin j holds e[j+1] < key <= e[j],
  // the last bin also key == e64
  int lo = 0, hi = kBins - 1;   // answer in [0, 63]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (e[mid] >= key) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(1024) topk_sample_kernel(TArgs a, StreamWs w) {
  extern __shared__ __align__(16) uint32_t sk[];   // kSamples keys
  const int r = blockIdx.x, tid = threadIdx.x;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  for (int e = tid; e < kSamples; e += 1024) {
    const int run = e / kSRun, o = e % kSRun;
    const int64_t pos = static_cast<int64_t>(run) * (a.n - kSRun) / (kSRuns - 1) + o;
    sk[e] = float_key(__ldg(row + pos));
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= kSamples; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < kSamples / 2; i += 1024) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint32_t x = sk[lo], y = sk[hi];
        if (desc ? (x < y) : (x > y)) {
          sk[lo] = y;
          sk[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  if (tid <= kBins) {
    const double p = static_cast<double>(a.k) / a.n;
    const double kp = p * kSamples;
    const double delta = 4.0 * sqrt(kSamples * p * (1.0 - p)) + 16.0;
    const double r_hi = kp - delta, r_lo = kp + delta;
    const double rank = r_hi + tid * (r_lo - r_hi) / kBins;
    const int ri = static_cast<int>(floor(rank));
    uint32_t e;
    if (tid == 0 && r_hi < 0.0) e = 0xFFFFFFFFu;
    else if (tid == kBins && r_lo >= kSamples - 1) e = 0u;
    else e = sk[min(max(ri, 0), kSamples - 1)];
    w.edges[static_cast<int64_t>(r) * (kBins + 1) + tid] = e;
  }
}

// block-wide exclusive scan for 512-thread CTAs (scratch [16])
__device__ __forceinline__ uint32_t scan512(uint32_t v, uint32_t* wt, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) wt[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < 16 ? wt[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += t;
    }
    if (lane < 16) wt[lane] = x;
  }
  __syncthreads();
  total = wt[15];
  const uint32_t pre = (warp > 0 ? wt[warp - 1] : 0u) + inc - v;
  __syncthreads();   // wt is reused by the caller's next scan
  return pre;
}

__global__ void __launch_bounds__(kCThreads2) topk_filter_kernel(TArgs a, StreamWs w) {
  __shared__ uint32_t e[kBins + 1];
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t wt[16];
  __shared__ uint32_t base_s;
  const int c = blockIdx.x, r = blockIdx.y, tid = threadIdx.x;
  if (tid <= kBins) e[tid] = w.edges[static_cast<int64_t>(r) * (kBins + 1) + tid];
  if (tid < kBins) hist[tid] = 0u;
  __syncthreads();
  const uint32_t e0 = e[0], e64 = e[kBins];
  const int64_t j0 = static_cast<int64_t>(c) * kChunk;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  // 32 keys per thread, coalesced: float4 q of thread t covers keys j0 + 4 (q * 512 + t) ..
  uint32_t key[32];
  int nan_local = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int64_t j = j0 + 4 * (static_cast<int64_t>(q) * kCThreads2 + tid);
    float f[4];
    if (j + 3 < a.n) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + j));
      f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) f[u] = j + u < a.n ? row[j + u] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      nan_local |= f[u] != f[u];
      key[4 * q + u] = j + u < a.n ? float_key(f[u]) : 0u;   // 0: below every bracket (e64 >= 0 ...)
    }
  }
  uint32_t gt = 0u, nc = 0u;
#pragma unroll
  for (int u = 0; u < 32; ++u) {
    const int64_t j = j0 + 4 * (static_cast<int64_t>(u >> 2) * kCThreads2 + tid) + (u & 3);
    const bool valid = j < a.n;
    gt += (valid && key[u] > e0) ? 1u : 0u;
    const bool cand = valid && key[u] <= e0 && key[u] >= e64;
    if (cand) {
      atomicAdd(&hist[bin_of(key[u], e)], 1u);
      ++nc;
    }
  }
  uint32_t tot_gt, tot_c;
  scan512(gt, wt, tot_gt);
  const uint32_t pre = scan512(nc, wt, tot_c);
  if (tid == 0) {
    w.chunk_gt[static_cast<int64_t>(r) * w.nchunk + c] = tot_gt;
    base_s = tot_c ? atomicAdd(&w.ccount[r], tot_c) : 0u;
  }
  __syncthreads();
  if (tid < kBins && hist[tid]) atomicAdd(&w.hist[static_cast<int64_t>(r) * kBins + tid], hist[tid]);
  if (nan_local) report(a.status, SPATTEN_E_NONFINITE);
  const uint32_t base = base_s;
  if (base + tot_c <= static_cast<uint32_t>(w.cap) && nc) {
    uint2* dst = w.cand + static_cast<int64_t>(r) * w.cap + base + pre;
    uint32_t m = 0u;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int64_t j = j0 + 4 * (static_cast<int64_t>(u >> 2) * kCThreads2 + tid) + (u & 3);
      if (j < a.n && key[u] <= e0 && key[u] >= e64) dst[m++] = make_uint2(key[u], static_cast<uint32_t>(j));
    }
  }
}

__global__ void __launch_bounds__(1024) topk_resolve_kernel(TArgs a, StreamWs w) {
  extern __shared__ __align__(16) unsigned char rs_smem[];
  uint64_t* bc = reinterpret_cast<uint64_t*>(rs_smem);                   // [kBinCap] sub-bin candidates
  uint32_t* cnt = reinterpret_cast<uint32_t*>(bc + kBinCap);             // [nchunk]
  __shared__ uint32_t e[kBins + 1];
  __shared__ uint32_t red[2][2][32];
  __shared__ uint32_t n_bc, jstar_s, above_s, ok_s;
  __shared__ uint32_t gt_part[32];
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid <= kBins) e[tid] = w.edges[static_cast<int64_t>(r) * (kBins + 1) + tid];
  if (tid == 0) n_bc = 0u;
  // total above the bracket
  uint32_t g = 0u;
  for (int c = tid; c < w.nchunk; c += 1024) {
    const uint32_t x = w.chunk_gt[static_cast<int64_t>(r) * w.nchunk + c];
    cnt[c] = x;
    g += x;
  }
  g = __reduce_add_sync(0xffffffffu, g);
  if (lane == 0) gt_part[warp] = g;
  __syncthreads();
  if (tid == 0) {
    uint32_t total_gt = 0u;
    for (int i = 0; i < 32; ++i) total_gt += gt_part[i];
    const uint32_t ncand = w.ccount[r];
    const uint32_t k = static_cast<uint32_t>(a.k);
    uint32_t ok = ncand <= static_cast<uint32_t>(w.cap) && total_gt < k && k <= total_gt + ncand;
    uint32_t acc = total_gt, js = kBins;
    if (ok) {
      for (int j = 0; j < kBins; ++j) {
        const uint32_t hj = w.hist[static_cast<int64_t>(r) * kBins + j];
        if (acc + hj >= k) { js = j; break; }
        acc += hj;
      }
      if (js == kBins || w.hist[static_cast<int64_t>(r) * kBins + js] > kBinCap) ok = 0u;
    }
    jstar_s = js;
    above_s = acc;
    ok_s = ok;
  }
  __syncthreads();
  const uint32_t ncand = w.ccount[r];
  if (!ok_s) {   // uniform
    if (tid == 0) {
      w.fallback[r] = 1;
      w.res[static_cast<int64_t>(r) * 4] = 0u;
    }
    return;
  }
  // the sub-bin's candidates as (key, ~index) composites
  const int js = static_cast<int>(jstar_s);
  const uint2* cand = w.cand + static_cast<int64_t>(r) * w.cap;
  for (uint32_t i = tid; i < ncand; i += 1024) {
    const uint2 cd = cand[i];
    if (bin_of(cd.x, e) == js) {
      const uint32_t slot = atomicAdd(&n_bc, 1u);
      if (slot < kBinCap) bc[slot] = (static_cast<uint64_t>(cd.x) << 32) | static_cast<uint64_t>(~cd.y);
    }
  }
  __syncthreads();
  const uint32_t m = min(n_bc, static_cast<uint32_t>(kBinCap));
  const uint32_t need = static_cast<uint32_t>(a.k) - above_s;   // 1 <= need <= m
  uint64_t v[kBinCap / 1024];
#pragma unroll
  for (int u = 0; u < kBinCap / 1024; ++u) {
    const uint32_t i = tid + u * 1024;
    v[u] = i < m ? bc[i] : 0ull;   // 0 lies below every candidate composite used as a threshold
  }
  // T = the need-th largest composite, two bits per round (the largest T with count(>= T) >= need)
  uint64_t T = 0ull;
  int rnd = 0;
#pragma unroll 1
  for (int b = 62; b >= 0; b -= 2, ++rnd) {
    const uint64_t c1 = T | (1ull << b), c2 = T | (2ull << b), c3 = T | (3ull << b);
    uint32_t x = 0u, y = 0u;
#pragma unroll
    for (int u = 0; u < kBinCap / 1024; ++u) {
      x += (v[u] >= c1 ? 1u : 0u) + (v[u] >= c2 ? 0x10000u : 0u);
      y += v[u] >= c3 ? 1u : 0u;
    }
    x = __reduce_add_sync(0xffffffffu, x);
    y = __reduce_add_sync(0xffffffffu, y);
    if (lane == 0) {
      red[rnd & 1][0][warp] = x;
      red[rnd & 1][1][warp] = y;
    }
    __syncthreads();
    x = 0u;
    y = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      x += red[rnd & 1][0][i];
      y += red[rnd & 1][1][i];
    }
    const uint32_t n1 = x & 0xFFFFu, n2 = x >> 16, n3 = y;
    T |= static_cast<uint64_t>((n1 >= need) + (n2 >= need) + (n3 >= need)) << b;
  }
  const uint32_t t_key = static_cast<uint32_t>(T >> 32), t_idx = ~static_cast<uint32_t>(T);
  // chunk offsets: above the bracket plus the selected candidates of each chunk
  for (uint32_t i = tid; i < ncand; i += 1024) {
    const uint2 cd = cand[i];
    if (cd.x > t_key || (cd.x == t_key && cd.y <= t_idx)) atomicAdd(&cnt[cd.y / kChunk], 1u);
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t acc = 0u;
    for (int c = 0; c < w.nchunk; ++c) {
      w.chunk_off[static_cast<int64_t>(r) * w.nchunk + c] = acc;
      acc += cnt[c];
    }
    uint32_t* rr = w.res + static_cast<int64_t>(r) * 4;
    rr[0] = 1u;
    rr[1] = t_key;
    rr[2] = t_idx;
    w.fallback[r] = 0;
  }
}

__global__ void __launch_bounds__(kCThreads2) topk_output_kernel(TArgs a, StreamWs w) {
  __shared__ uint32_t wt[16];
  const int c = blockIdx.x, r = blockIdx.y, tid = threadIdx.x;
  const uint32_t* rr = w.res + static_cast<int64_t>(r) * 4;
  if (!rr[0]) return;   // uniform: the row is redone by the fallback
  const uint32_t t_key = rr[1], t_idx = rr[2];
  // 32 consecutive keys per thread (index order within the thread)
  const int64_t j0 = static_cast<int64_t>(c) * kChunk + tid * 32;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  uint32_t sel = 0u;   // bit u: key j0 + u selected
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int64_t j = j0 + 4 * q;
    float f[4];
    if (j + 3 < a.n) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + j));
      f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) f[u] = j + u < a.n ? row[j + u] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t key = float_key(f[u]);
      const bool s = j + u < a.n && (key > t_key || (key == t_key && static_cast<uint32_t>(j + u) <= t_idx));
      sel |= (s ? 1u : 0u) << (4 * q + u);
    }
  }
  uint32_t total;
  const uint32_t pre = scan512(__popc(sel), wt, total);
  uint32_t pos = w.chunk_off[static_cast<int64_t>(r) * w.nchunk + c] + pre;
  int32_t* out = a.idx_out + static_cast<int64_t>(r) * a.ld_out;
  while (sel) {
    const int u = __ffs(sel) - 1;
    sel &= sel - 1u;
    if (pos < static_cast<uint32_t>(a.k)) out[pos] = static_cast<int32_t>(j0 + u);
    ++pos;
  }
}

int stream_cap(int n) { return std::max(4096, n / 16); }

bool stream_applicable(const TArgs& a) {
  return a.map == nullptr && a.idx_out != nullptr && a.n >= kStreamMin && a.k > 0 && a.k < a.n &&
         (a.ld & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
}

size_t stream_ws_bytes(int R, int n) {
  const size_t nchunk = (static_cast<size_t>(n) + kChunk - 1) / kChunk;
  size_t b = 0;
  auto take = [&](size_t bytes) { b += (bytes + 255) & ~size_t(255); };
  take(static_cast<size_t>(R) * kBins * 4);            // hist (zeroed)
  take(static_cast<size_t>(R) * 4);                    // ccount (zeroed)
  take(static_cast<size_t>(R) * (kBins + 1) * 4);      // edges
  take(static_cast<size_t>(R) * nchunk * 4);           // chunk_gt
  take(static_cast<size_t>(R) * nchunk * 4);           // chunk_off
  take(static_cast<size_t>(R) * 16);                   // res
  take(static_cast<size_t>(R) * 4);                    // fallback
  take(static_cast<size_t>(R) * stream_cap(n) * 8);    // cand
  return b;
}

int pick_cluster(int n) {
  // one CTA per 4096 keys, at most 8 (portable cluster size); the launcher may widen very long
  // rows to 16 when the device can schedule such clusters
  int C = static_cast<int>(ceil_div(n, 4096));
  return std::max(1, std::min(C, 8));
}

}  // namespace

bool stream_fits(int R, int n) {
  (void)R;
  return n >= kStreamMin && (static_cast<int64_t>(n) + kChunk - 1) / kChunk <= 8192;
}

size_t topk_workspace_bytes(int R, int n, int k) {
  (void)k;
  return stream_fits(R, n) ? stream_ws_bytes(R, n) : 0;
}

int32_t cluster_launch(const TArgs& a, cudaStream_t st);

int32_t topk_stream_launch(const TArgs& a, void* ws, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  SPT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return SPATTEN_E_UNSUPPORTED;
  if (!configured[dev]) {
    SPT_CUDA(cudaFuncSetAttribute(topk_sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSamples * 4));
    SPT_CUDA(cudaFuncSetAttribute(topk_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kBinCap * 8 + 8192 * 4));
    configured[dev] = true;
  }
  const int R = a.R, n = a.n;
  StreamWs w{};
  w.nchunk = static_cast<int>((static_cast<int64_t>(n) + kChunk - 1) / kChunk);
  w.cap = stream_cap(n);
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t bytes) {
    char* q = p;
    p += (bytes + 255) & ~size_t(255);
    return q;
  };
  w.hist = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * kBins * 4));
  w.ccount = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * 4));
  const size_t zero_bytes = static_cast<size_t>(p - static_cast<char*>(ws));
  w.edges = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * (kBins + 1) * 4));
  w.chunk_gt = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * w.nchunk * 4));
  w.chunk_off = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * w.nchunk * 4));
  w.res = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * 16));
  w.fallback = reinterpret_cast<int32_t*>(take(static_cast<size_t>(R) * 4));
  w.cand = reinterpret_cast<uint2*>(take(static_cast<size_t>(R) * w.cap * 8));
  SPT_CUDA(cudaMemsetAsync(ws, 0, zero_bytes, st));
  topk_sample_kernel<<<R, 1024, kSamples * 4, st>>>(a, w);
  SPT_TRY(launch_status());
  topk_filter_kernel<<<dim3(w.nchunk, R), kCThreads2, 0, st>>>(a, w);
  SPT_TRY(launch_status());
  topk_resolve_kernel<<<R, 1024, static_cast<size_t>(kBinCap) * 8 + static_cast<size_t>(w.nchunk) * 4, st>>>(a, w);
  SPT_TRY(launch_status());
  topk_output_kernel<<<dim3(w.nchunk, R), kCThreads2, 0, st>>>(a, w);
  SPT_TRY(launch_status());
  TArgs f = a;   // rows whose bracket missed: the cluster kernel, every other row skipped at once
  f.only_rows = w.fallback;
  return cluster_launch(f, st);
}

int32_t topk_launch(const TArgs& a, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (stream_applicable(a) && stream_fits(a.R, a.n) && ws && ws_bytes >= stream_ws_bytes(a.R, a.n))
    return topk_stream_launch(a, ws, st);
  if (a.n <= 32 * kSKeys) {
    topk_small_kernel<1><<<static_cast<unsigned>(ceil_div(a.R, 4)), 128, 0, st>>>(a);
    return launch_status();
  }
  if (a.n <= 128 * kSKeys) {
    topk_small_kernel<4><<<a.R, 128, 0, st>>>(a);
    return launch_status();
  }
  if (a.n <= 512 * kSKeys) {
    topk_small_kernel<16><<<a.R, 512, 0, st>>>(a);
    return launch_status();
  }
  return cluster_launch(a, st);
}

int32_t cluster_launch(const TArgs& a, cudaStream_t st) {
  static bool configured[64] = {false};
  static bool wide_ok[64] = {false};   // 16-CTA clusters can be scheduled on this device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    SPT_CUDA(cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kResident * 4));
    if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(16, 1, 1);
      q.blockDim = dim3(kTThreads, 1, 1);
      q.dynamicSmemBytes = kResident * 4;
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = 16;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.attrs = qa;
      q.numAttrs = 1;
      int clusters = 0;
      wide_ok[dev] = cudaOccupancyMaxActiveClusters(&clusters, topk_cluster_kernel, &q) == cudaSuccess && clusters >= 4;
    }
    cudaGetLastError();   // the probe above may leave an error behind
    configured[dev] = true;
  }
  int C = pick_cluster(a.n);
  if (C == 8 && a.n > 8 * kResident && dev >= 0 && dev < 64 && wide_ok[dev]) C = 16;
  const int chunk = static_cast<int>((ceil_div(a.n, C) + 3) & ~int64_t(3));
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
  if (!scores || (!idx_out && !comp_out)) return SPATTEN_E_ARG;
  if (R < 1 || n < 1 || k < 0 || R > 65535) return SPATTEN_E_ARG;
  if (k > n) return SPATTEN_E_SHAPE;
  if (ld_out < k) return SPATTEN_E_SHAPE;
  if (!map && ld < n) return SPATTEN_E_SHAPE;
  if (map && ld_map < n) return SPATTEN_E_SHAPE;
  if (comp_out && !map) return SPATTEN_E_ARG;
  TArgs a{scores, R, n, ld, k, map, ld_map, idx_out, ld_out, comp_out, dev_status};
  return topk_launch(a, ws, ws_bytes, as_stream(stream));
}
