// K4: batched top-k selection with a deterministic tie-break and ascending-index output.
//
// SpAtten §IV.B "Top-k Engine" avoids a full sort: it finds the k-th largest value as a threshold
// with quick-select, filters the array against it and removes the gaps with a prefix-sum-driven
// zero eliminator.  The B200 forms of the same three steps, by row length:
//   n <= 8192      (topk_small_kernel) the row's order-preserving 32-bit keys live in registers;
//                  the threshold is a two-bits-per-round digit search with warp reductions; one
//                  packed block scan places every kept key.
//   longer rows    (topk_cluster_kernel) radix select over the keys: four 8-bit digit passes, each
//                  a shared-memory histogram of the keys that still match the known high digits;
//                  the CTAs of a thread-block cluster (one cluster per row) add their histograms
//                  through distributed shared memory.  Each CTA keeps up to kResident keys of its
//                  chunk in shared memory; the rest is streamed again from L2 in every pass.
//   n >= 65536 with the caller's workspace (sample / filter / resolve / output kernels): a
//                  sampled rank window around the k-th key, one streaming pass that marks the keys
//                  above the window in a bit mask and collects the window's keys, an exact select among those
//                  candidates, an output pass over that pass's bit mask (see the section below).
// In every form a key is kept if it is above the threshold T, or equal to T and among the first
// (k - #above) equal keys in index order (ties go to the lower index), and warp ballots / block
// scans give each kept key its output slot in ascending index order.
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

// one row for one cluster; every CTA of the cluster calls it with the same row
__device__ __forceinline__ void cluster_row(const TArgs& a, int r, uint32_t* keys_s, TShared& sh) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

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

// row blockIdx.y; LOOP: rows blockIdx.y, blockIdx.y + gridDim.y, ... (each row's last cluster
// barrier ends every read of a peer's shared memory for that row, so the next row may reuse it)
template <bool LOOP>
__global__ void __launch_bounds__(kTThreads) topk_cluster_kernel(TArgs a) {
  extern __shared__ __align__(16) uint32_t keys_s[];
  __shared__ TShared sh;
  if (LOOP) {
    for (int r = blockIdx.y; r < a.R; r += gridDim.y) cluster_row(a, r, keys_s, sh);
  } else {
    cluster_row(a, blockIdx.y, keys_s, sh);
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
// Long rows (n >= kStreamMin, scores read directly, caller workspace given): one streaming pass
// over the scores between a sample and an exact select on small data (one CTA per row each), then
// an output pass over the pass's bit mask and candidates.
//  sample   one CTA per row draws 16 K keys (64 evenly spaced runs of 256; 8 K keys in runs of 128
//           for rows under 512 K keys) and finds by a digit search the sample keys e0 >= e64 at
//           the two ends of a rank window around the sample rank of the k-th key (+-4 sigma of the
//           sampling error + 16; an end past the sample is left open).  The search runs first on
//           each thread's first key (one in 16, or in 8), whose own window, widened by its
//           sampling error, bounds the few thousand sample keys the exact search then needs.  It
//           also fixes the sub-bin scale: 64 steps of equal width in value between the window's
//           ends (the sample's extreme key in place of an open end).
//  filter   per chunk of 8 K keys: the keys above e0 (a count and a bit mask), the keys in
//           [e64, e0] appended as (score bits, index) to the row's candidate list, and their
//           histogram over the 64 sub-bins
//  resolve  one CTA per row: the sub-bin holding the k-th key, the exact threshold among that
//           sub-bin's candidates as the (need)-th largest (key, ~index) composite (ties to the lower
//           index), and every chunk's output offset.  It also sets the mask bits of the selected
//           candidates: every candidate of the sub-bins above T's, and T's own selected part.
//  output   per chunk: the indices of the mask's set bits, written in index order (the scores are
//           not read again)
// A row whose k-th key fell outside the window, or whose buffers overflowed, is marked and done
// again by the cluster kernel (only_rows).
// The filter reads a warp's 512 keys as four coalesced 16-byte loads per lane (load q of lane t
// holds keys 128 q + 4 t .. 128 q + 4 t + 3 of the warp's span) and compares floats against the
// window ends turned back into floats (the key map is monotone, and -0.0 equals +0.0 on both
// sides); a NaN fails every ordered comparison, lands in the candidate list and is reported by the
// resolve step.  Its above-window bits go out in index order, one 32-bit word per 32 keys; the
// resolve step adds the selected candidates' bits, and the output step turns each word into
// indices.
// ------------------------------------------------------------------------------------------------
constexpr int kStreamMin = 65536;
constexpr int kSRuns = 64;                                              // sample runs per row
constexpr int kBins = 64;
constexpr int kRThreads = 1024;                                         // sample and resolve CTAs
constexpr int kFThreads = 512;                                          // filter and output CTAs
constexpr int kFWarps = kFThreads / 32;
constexpr int kFKeys = 16;                                              // keys per filter/output lane
constexpr int kChunk = kFThreads * kFKeys;                              // 8 K keys per filter/output CTA
constexpr int kBinCap = 8192;                                           // candidates of one sub-bin
constexpr int kL1 = 1024;                                               // first-level sample keys
// the sample of one row: KPT keys per thread of a 1024-thread CTA, in 64 runs of 16 threads'
// keys; the second-level list holds a quarter of the sample.  16 K keys (KPT 16) for rows of
// 512 K keys and more, 8 K (KPT 8) below: a smaller sample costs a wider window (more candidates
// for the filter and resolve steps), which pays off only where the sample step is a large share
template <int KPT>
struct SampleCfg {
  static constexpr int kSRun = 16 * KPT;                 // keys per run
  static constexpr int kSamples = kSRuns * kSRun;        // sample keys per row
  static constexpr int kSList = kSamples / 4;            // second-level sample keys
};
constexpr int kMaxChunks = 8192;

struct StreamWs {
  float* ends;          // [R][4]     window ends e0 (top), e64 (bottom) for the tests (+-inf when
                        //            open), and the sub-bin scale's top and 64 / width (its ends
                        //            the sample's extreme key in place of an open end)
  uint32_t* ccount;     // [R]        candidates appended (zeroed by the sample kernel)
  uint32_t* chunk_gt;   // [R][nchunk]
  uint32_t* hist;       // [R][nchunk][kBins]   candidates of each chunk per sub-bin
  uint2* cand;          // [R][cap]  (score bits, index)
  uint32_t* chunk_off;  // [R][nchunk]
  uint32_t* gtmask;     // [R][nchunk][kChunk / 32]  bit j % 32 of word j / 32 (row key j): above the
                        //            window (filter), or a selected candidate (resolve)
  uint32_t* res;        // [R][4]   valid, T key, T index, spare
  int32_t* fallback;    // [R]
  int cap, nchunk;
};

// float of a key (the inverse of float_key); the keys of NaNs, which only the window's special
// ends use, give +-infinity
__device__ __forceinline__ float key_float(uint32_t k) {
  if (k > 0xFF800000u) return __int_as_float(0x7F800000);
  if (k <= 0x007FFFFFu) return __int_as_float(static_cast<int>(0xFF800000u));
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// sub-bin of a window value: 64 steps of equal width from the scale's top down to its bottom
// (clamped at both ends; all in sub-bin 0 when an end is infinite); the same rounded operations on
// both sides of the candidate list, so the filter and the resolve step agree bit for bit; monotone
// in the value
struct BinMap {
  float top, inv;
};

__device__ __forceinline__ BinMap bin_map(float fe0, float fe64) {
  const float span = __fsub_rn(fe0, fe64);
  const bool ok = fabsf(fe0) <= 3.402823466e38f && fabsf(fe64) <= 3.402823466e38f && span > 0.0f;
  return {fe0, ok ? __fdiv_rn(static_cast<float>(kBins), span) : 0.0f};
}

__device__ __forceinline__ int bin_of(float f, const BinMap& m) {
  const int b = __float2int_rz(__fmul_rn(__fsub_rn(m.top, f), m.inv));
  return min(max(b, 0), kBins - 1);
}

// Programmatic dependent launch between the streaming steps: the filter, resolve and output
// kernels are launched with programmatic stream serialisation, so their CTAs may start while the
// previous step still runs (every CTA of that step is resident by then: each one triggers at its
// start).  grid_dep_wait() returns once the previous step's grid has completed and its writes are
// visible; nothing that step writes is read before it.  The filter issues its score loads (input
// only) before the wait, beside the sample step.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// bitonic sort of one value per thread over a 1024-thread block, descending (thread t ends with
// sorted position t); partners closer than a warp exchange by shuffles, the others through
// `scratch` [1024]; every thread must call it, and scratch is free again after a block barrier
template <typename V>
__device__ __forceinline__ V bitonic_desc_1024(V x, V* scratch) {
  const int tid = threadIdx.x;
  for (int size = 2; size <= 1024; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      V y;
      if (stride >= 32) {
        __syncthreads();
        scratch[tid] = x;
        __syncthreads();
        y = scratch[tid ^ stride];
      } else {
        y = __shfl_xor_sync(0xffffffffu, x, stride);
      }
      const bool lower = (tid & stride) == 0, desc = (tid & size) == 0;
      const bool take_max = lower == desc;
      x = take_max ? (x > y ? x : y) : (x < y ? x : y);
    }
  }
  return x;
}

template <int KPT>
struct SampleSmem {
  uint32_t red[2][3][32];
  uint32_t cnt[32];
  uint32_t list[SampleCfg<KPT>::kSList];
  int rank[2];        // sample ranks of the window's ends
  int open[2];        // the window's top / bottom end lies past the sample
  int l1[2];          // first-level ranks of the outer bounds (< 0 / >= kL1: no bound)
  uint32_t n_list;
};

// ta / tb = the need_a-th / need_b-th largest of the NK keys per thread (block-wide; padding keys
// are 0 and never counted): the largest T with count(>= T) >= need, two bits per round; counts fit
// 16 bits (at most 16 K), two per word.  While the two share their high bits one set of three
// counts serves both.
template <int NK, class SM>
__device__ __forceinline__ void search2(const uint32_t* key, uint32_t need_a, uint32_t need_b, SM& sm,
                                        uint32_t& ta, uint32_t& tb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  ta = 0u;
  tb = 0u;
  int rnd = 0;
#pragma unroll 1
  for (int b = 30; b >= 0; b -= 2, ++rnd) {
    const bool same = ta == tb;   // uniform
    const uint32_t a1 = ta | (1u << b), a2 = ta | (2u << b), a3 = ta | (3u << b);
    const uint32_t b1 = tb | (1u << b), b2 = tb | (2u << b), b3 = tb | (3u << b);
    uint32_t x = 0u, y = 0u, z = 0u;
    if (same) {
#pragma unroll
      for (int i = 0; i < NK; ++i) {
        x += (key[i] >= a1 ? 1u : 0u) + (key[i] >= a2 ? 0x10000u : 0u);
        y += key[i] >= a3 ? 1u : 0u;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NK; ++i) {
        x += (key[i] >= a1 ? 1u : 0u) + (key[i] >= a2 ? 0x10000u : 0u);
        y += (key[i] >= a3 ? 1u : 0u) + (key[i] >= b1 ? 0x10000u : 0u);
        z += (key[i] >= b2 ? 1u : 0u) + (key[i] >= b3 ? 0x10000u : 0u);
      }
    }
    x = __reduce_add_sync(0xffffffffu, x);
    y = __reduce_add_sync(0xffffffffu, y);
    z = __reduce_add_sync(0xffffffffu, z);
    if (lane == 0) {
      sm.red[rnd & 1][0][warp] = x;
      sm.red[rnd & 1][1][warp] = y;
      sm.red[rnd & 1][2][warp] = z;
    }
    __syncthreads();
    x = __reduce_add_sync(0xffffffffu, sm.red[rnd & 1][0][lane]);
    y = __reduce_add_sync(0xffffffffu, sm.red[rnd & 1][1][lane]);
    z = __reduce_add_sync(0xffffffffu, sm.red[rnd & 1][2][lane]);
    const uint32_t n1 = x & 0xFFFFu, n2 = x >> 16, n3 = y & 0xFFFFu;
    ta |= static_cast<uint32_t>((n1 >= need_a) + (n2 >= need_a) + (n3 >= need_a)) << b;
    if (same) tb |= static_cast<uint32_t>((n1 >= need_b) + (n2 >= need_b) + (n3 >= need_b)) << b;
    else tb |= static_cast<uint32_t>(((y >> 16) >= need_b) + ((z & 0xFFFFu) >= need_b) + ((z >> 16) >= need_b)) << b;
  }
}

// append the keys with in == true to `list` (warp-aggregated slots; at most cap kept)
__device__ __forceinline__ void append_keys(bool in, uint32_t key, uint32_t* list, uint32_t* n, uint32_t cap) {
  const int lane = threadIdx.x & 31;
  const uint32_t m = __ballot_sync(0xffffffffu, in);
  if (m) {
    const int leader = __ffs(m) - 1;
    uint32_t base = 0u;
    if (lane == leader) base = atomicAdd(n, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    const uint32_t s = base + __popc(m & ((1u << lane) - 1u));
    if (in && s < cap) list[s] = key;
  }
}

// the window's ends from the NK keys per thread, which hold every sample key ranked in the window;
// `base` more sample keys lie above all of them
template <int NK, class SM>
__device__ __forceinline__ void window_ends(const uint32_t* key, uint32_t base, SM& sm, int r, StreamWs& w) {
  const uint32_t need_a = static_cast<uint32_t>(sm.rank[0]) + 1u - base;
  const uint32_t need_b = static_cast<uint32_t>(sm.rank[1]) + 1u - base;
  uint32_t ta, tb;
  search2<NK>(key, need_a, need_b, sm, ta, tb);
  if (threadIdx.x == 0) {   // with an open end, ta / tb are the sample's largest / smallest key
    const BinMap bm = bin_map(key_float(ta), key_float(tb));
    w.ends[4 * r] = key_float(sm.open[0] ? 0xFFFFFFFFu : ta);
    w.ends[4 * r + 1] = key_float(sm.open[1] ? 0u : tb);
    w.ends[4 * r + 2] = bm.top;
    w.ends[4 * r + 3] = bm.inv;
  }
}

template <int KPT>
__global__ void __launch_bounds__(kRThreads) topk_sample_kernel(TArgs a, StreamWs w) {
  constexpr int kSRun = SampleCfg<KPT>::kSRun, kSamples = SampleCfg<KPT>::kSamples, kSList = SampleCfg<KPT>::kSList;
  static_assert(kSamples == KPT * kRThreads, "KPT sample keys per thread");
  static_assert(kL1 == kRThreads, "one first-level key per thread");
  __shared__ SampleSmem<KPT> sm;
  grid_dep_trigger();
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  // thread t reads 16 consecutive keys of run t / 16 (runs start on a 16-byte boundary)
  uint32_t key[KPT];
  {
    const int run = tid / (kSRun / KPT);
    const int64_t pos = ((static_cast<int64_t>(run) * (a.n - kSRun) / (kSRuns - 1)) & ~int64_t(3)) +
                        (tid % (kSRun / KPT)) * KPT;
#pragma unroll
    for (int q = 0; q < KPT / 4; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + pos) + q);
      key[4 * q] = float_key(v.x);
      key[4 * q + 1] = float_key(v.y);
      key[4 * q + 2] = float_key(v.z);
      key[4 * q + 3] = float_key(v.w);
    }
  }
  if (tid == 0) {
    sm.n_list = 0u;
    w.ccount[r] = 0u;
  }
  if (tid < 2) {
    // sample ranks of the window's ends [r_hi, r_lo] around k/n of the sample
    const double p = static_cast<double>(a.k) / a.n;
    const double kp = p * kSamples;
    const double delta = 4.0 * sqrt(kSamples * p * (1.0 - p)) + 16.0;
    const double r_hi = kp - delta, r_lo = kp + delta;
    const int rho = min(max(static_cast<int>(floor(tid == 0 ? r_hi : r_lo)), 0), kSamples - 1);
    sm.rank[tid] = rho;
    sm.open[tid] = tid == 0 ? r_hi < 0.0 : r_lo >= kSamples - 1;
    // first level: one sample key in 16; its keys at the window ends' ranks, moved outwards by 4
    // sigma of their own rank error (in first-level ranks) + 8, bound a second-level set that holds
    // the window
    const int m1 = static_cast<int>(ceil(4.0 * sqrt(kL1 * p * (1.0 - p)) + 8.0));
    constexpr int kStep = kSamples / kL1;
    sm.l1[tid] = tid == 0 ? rho / kStep - m1 : (rho + kStep - 1) / kStep + m1;
  }
  __syncthreads();
  // the first level: each thread's first key, 16 per run
  uint32_t k1 = key[0];
  const int l1a = sm.l1[0], l1b = sm.l1[1];
  uint32_t ca, cb;
  search2<1>(&k1, static_cast<uint32_t>(max(l1a, 0)) + 1u, static_cast<uint32_t>(min(l1b, kL1 - 1)) + 1u, sm, ca, cb);
  if (l1a < 0) ca = 0xFFFFFFFFu;
  if (l1b >= kL1) cb = 0u;
  // the bound holds if at most rank[0] sample keys exceed ca and at least rank[1] + 1 reach cb
  uint32_t c = 0u;
#pragma unroll
  for (int i = 0; i < KPT; ++i) c += (key[i] > ca ? 1u : 0u) + (key[i] >= cb ? 0x10000u : 0u);
  c = __reduce_add_sync(0xffffffffu, c);
  if (lane == 0) sm.cnt[warp] = c;
  __syncthreads();
  c = __reduce_add_sync(0xffffffffu, sm.cnt[lane]);
  const uint32_t gt_ca = c & 0xFFFFu, ge_cb = c >> 16;
  const bool narrow = gt_ca <= static_cast<uint32_t>(sm.rank[0]) && ge_cb >= static_cast<uint32_t>(sm.rank[1]) + 1u &&
                      ge_cb - gt_ca <= static_cast<uint32_t>(kSList);   // uniform
  if (narrow) {
#pragma unroll
    for (int i = 0; i < KPT; ++i) append_keys(key[i] >= cb && key[i] <= ca, key[i], sm.list, &sm.n_list, kSList);
    __syncthreads();
    constexpr int NL = kSList / kRThreads;
    uint32_t s[NL];
    const uint32_t nl = sm.n_list;
#pragma unroll
    for (int u = 0; u < NL; ++u) s[u] = tid + u * kRThreads < static_cast<int>(nl) ? sm.list[tid + u * kRThreads] : 0u;
    window_ends<NL>(s, gt_ca, sm, r, w);
  } else {
    window_ends<KPT>(key, 0u, sm, r, w);
  }
}

// the kFKeys scores of one filter/output lane (see the layout note above); FULL: the whole span
// lies inside the row
template <bool FULL>
__device__ __forceinline__ void load_span(const float* row, int jw, int n, float* f) {
#pragma unroll
  for (int q = 0; q < kFKeys / 4; ++q) {
    const int j = jw + 128 * q;
    if (FULL || j + 3 < n) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + j));
      f[4 * q] = v.x; f[4 * q + 1] = v.y; f[4 * q + 2] = v.z; f[4 * q + 3] = v.w;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) f[4 * q + u] = j + u < n ? row[j + u] : 0.0f;
    }
  }
}

__device__ __forceinline__ int span_off(int u) { return 128 * (u >> 2) + (u & 3); }

// the above-window mask (bit u: f[u] > fe0) and the candidate mask (bit u: f[u] in [fe64, fe0],
// or NaN) of one lane's kFKeys keys
template <bool FULL>
__device__ __forceinline__ void filter_span(const float* f, int jw, int n, float fe0, float fe64, uint32_t& gm,
                                            uint32_t& cm) {
  gm = 0u;
  cm = 0u;
#pragma unroll
  for (int u = 0; u < kFKeys; ++u) {
    if (FULL || span_off(u) < n - jw) {
      if (f[u] > fe0) gm |= 1u << u;
      if (!(f[u] < fe64 || f[u] > fe0)) cm |= 1u << u;
    }
  }
}

__global__ void __launch_bounds__(kFThreads, 4) topk_filter_kernel(TArgs a, StreamWs w) {
  __shared__ uint32_t wc[kFWarps], wg[kFWarps], wb[kFWarps];
  __shared__ uint32_t hist[kBins];
  const int c = blockIdx.x, r = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kBins) hist[tid] = 0u;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  const int jw = c * kChunk + warp * (32 * kFKeys) + 4 * lane;
  const int64_t rc = static_cast<int64_t>(r) * w.nchunk + c;
  const bool full = (c + 1) * kChunk <= a.n;
  float f[kFKeys];
  if (full) load_span<true>(row, jw, a.n, f);
  else load_span<false>(row, jw, a.n, f);
  grid_dep_trigger();
  grid_dep_wait();   // the window ends and the zeroed candidate count come from the sample step
  const float4 en = reinterpret_cast<const float4*>(w.ends)[r];
  const float fe0 = en.x, fe64 = en.y;
  const BinMap bm{en.z, en.w};
  uint32_t gm, cm;
  if (full) filter_span<true>(f, jw, a.n, fe0, fe64, gm, cm);
  else filter_span<false>(f, jw, a.n, fe0, fe64, gm, cm);
  {
    // load q of lanes 8 g .. 8 g + 7 covers word 4 q + g of the warp's 16 (32 keys each), lane
    // 8 g + i at bits 4 i .. 4 i + 3
    uint32_t* dst = w.gtmask + rc * (kChunk / 32) + warp * kFKeys;
#pragma unroll
    for (int q = 0; q < kFKeys / 4; ++q) {
      uint32_t v = ((gm >> (4 * q)) & 0xFu) << (4 * (lane & 7));
      v |= __shfl_xor_sync(0xffffffffu, v, 1);
      v |= __shfl_xor_sync(0xffffffffu, v, 2);
      v |= __shfl_xor_sync(0xffffffffu, v, 4);
      if ((lane & 7) == 0) dst[4 * q + (lane >> 3)] = v;
    }
  }
  uint32_t gt = __popc(gm);
  const uint32_t nc = __popc(cm);
  uint32_t inc = nc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  gt = __reduce_add_sync(0xffffffffu, gt);
  if (lane == 31) wc[warp] = inc;
  if (lane == 0) wg[warp] = gt;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < kFWarps ? wc[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < kFWarps; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, xi, kFWarps - 1);
    const uint32_t g = __reduce_add_sync(0xffffffffu, lane < kFWarps ? wg[lane] : 0u);
    uint32_t base = 0u;
    if (lane == 0) {
      w.chunk_gt[rc] = g;
      if (tot) base = atomicAdd(&w.ccount[r], tot);
    }
    base = __shfl_sync(0xffffffffu, base, 0);
    // a chunk whose candidates would pass the list's end writes none (the row falls back)
    if (lane < kFWarps) wb[lane] = base + tot <= static_cast<uint32_t>(w.cap) ? base + xi - x : 0xFFFFFFFFu;
  }
  __syncthreads();
  const uint32_t wbase = wb[warp];
  if (wbase != 0xFFFFFFFFu) {
    uint2* dst = w.cand + static_cast<int64_t>(r) * w.cap + wbase + (inc - nc);
    // each candidate's score read again (an L1 hit) rather than held across the barriers
    uint32_t i = 0u;
    for (uint32_t mm = cm; mm; mm &= mm - 1u, ++i) {
      const int u = __ffs(mm) - 1;
      const int j = jw + 128 * (u >> 2) + (u & 3);
      const float f = row[j];
      dst[i] = make_uint2(__float_as_uint(f), static_cast<uint32_t>(j));
      atomicAdd(&hist[bin_of(f, bm)], 1u);
    }
  }
  __syncthreads();
  if (tid < kBins) w.hist[rc * kBins + tid] = hist[tid];
}

// exclusive prefix sum over a 1024-thread block (part: [32] scratch, free again after return)
__device__ __forceinline__ uint32_t scan1024(uint32_t v, uint32_t* part, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) part[warp] = inc;
  __syncthreads();
  const uint32_t p = part[lane];
  uint32_t pi = p;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, pi, o);
    if (lane >= o) pi += t;
  }
  total = __shfl_sync(0xffffffffu, pi, 31);
  const uint32_t before = __shfl_sync(0xffffffffu, pi - p, warp);
  __syncthreads();
  return before + inc - v;
}

__device__ __forceinline__ void stream_fail(StreamWs& w, int r) {
  if (threadIdx.x == 0) {
    w.fallback[r] = 1;
    w.res[static_cast<int64_t>(r) * 4] = 0u;
  }
}

__global__ void __launch_bounds__(kRThreads) topk_resolve_kernel(TArgs a, StreamWs w) {
  constexpr int BP = 8;   // (key, index) pairs per thread per batch
  extern __shared__ __align__(16) unsigned char rs_smem[];
  uint64_t* bc = reinterpret_cast<uint64_t*>(rs_smem);                   // [kBinCap] sub-bin candidates
  uint32_t* cnt = reinterpret_cast<uint32_t*>(bc + kBinCap);             // [nchunk]
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t red[2][2][32];
  __shared__ uint32_t part[32];
  __shared__ uint32_t n_bc, js_s, above_s;
  __shared__ uint64_t t_s;
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < kBins) hist[tid] = 0u;
  if (tid == 0) {
    n_bc = 0u;
    js_s = kBins;   // no sub-bin found: the row falls back
  }
  grid_dep_trigger();
  grid_dep_wait();   // everything below reads the filter step's results
  const int nchunk = w.nchunk;
  uint32_t g = 0u;
  for (int c = tid; c < nchunk; c += kRThreads) {
    const uint32_t x = w.chunk_gt[static_cast<int64_t>(r) * nchunk + c];
    cnt[c] = x;
    g += x;
  }
  g = __reduce_add_sync(0xffffffffu, g);
  if (lane == 0) part[warp] = g;
  __syncthreads();
  const uint32_t total_gt = __reduce_add_sync(0xffffffffu, part[lane]);
  const uint32_t ncand = w.ccount[r];
  const uint32_t k = static_cast<uint32_t>(a.k);
  if (!(ncand <= static_cast<uint32_t>(w.cap) && total_gt < k && k <= total_gt + ncand)) {   // uniform
    stream_fail(w, r);
    return;
  }
  // sub-bin totals from the chunks' histograms (thread: one sub-bin, every 16th chunk)
  const uint32_t* h = w.hist + static_cast<int64_t>(r) * nchunk * kBins;
  {
    const int j = tid & (kBins - 1), cg = tid / kBins;
    uint32_t s = 0u;
#pragma unroll 4
    for (int c = cg; c < nchunk; c += kRThreads / kBins) s += h[static_cast<int64_t>(c) * kBins + j];
    if (s) atomicAdd(&hist[j], s);
  }
  __syncthreads();
  if (warp == 0) {
    // the first sub-bin whose cumulative count reaches need = k - total_gt (>= 1; the sub-bins
    // hold all ncand >= need candidates, so exactly one lane finds it)
    const uint32_t need = k - total_gt;
    const uint32_t h0 = hist[2 * lane], h1 = hist[2 * lane + 1];
    uint32_t inc = h0 + h1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    const uint32_t ex = inc - h0 - h1;
    if (ex < need && ex + h0 >= need) {
      js_s = 2 * lane;
      above_s = total_gt + ex;
    } else if (ex + h0 < need && inc >= need) {
      js_s = 2 * lane + 1;
      above_s = total_gt + ex + h0;
    }
  }
  __syncthreads();
  const int js = static_cast<int>(js_s);
  if (js >= kBins || hist[js] > static_cast<uint32_t>(kBinCap)) {   // uniform
    stream_fail(w, r);
    return;
  }
  // the one pass over the candidate list: the sub-bins above js are selected whole (their mask
  // bits set), sub-bin js is collected as (key, ~index) composites; NaNs (they pass the filter) are
  // looked for on the way
  const BinMap bm{w.ends[4 * r + 2], w.ends[4 * r + 3]};
  const uint2* cand = w.cand + static_cast<int64_t>(r) * w.cap;
  uint32_t* mrow = w.gtmask + static_cast<int64_t>(r) * nchunk * (kChunk / 32);
  const uint32_t lt_mask = (1u << lane) - 1u;
  bool nan_seen = false;
  for (uint32_t i0 = 0; i0 < ncand; i0 += BP * kRThreads) {
    uint2 cd[BP];
#pragma unroll
    for (int u = 0; u < BP; ++u) {
      const uint32_t i = i0 + tid + u * kRThreads;
      cd[u] = i < ncand ? cand[i] : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < BP; ++u) {
      const float f = __uint_as_float(cd[u].x);
      nan_seen |= f != f;
      const bool live = i0 + tid + u * kRThreads < ncand;
      const int b = bin_of(f, bm);
      if (live && b < js) atomicOr(&mrow[cd[u].y >> 5], 1u << (cd[u].y & 31u));
      const bool hit = live && b == js;
      const uint32_t m = __ballot_sync(0xffffffffu, hit);
      if (m) {
        const int leader = __ffs(m) - 1;
        uint32_t base = 0u;
        if (lane == leader) base = atomicAdd(&n_bc, __popc(m));
        base = __shfl_sync(0xffffffffu, base, leader);
        const uint32_t slot = base + __popc(m & lt_mask);
        if (hit && slot < kBinCap) bc[slot] = (static_cast<uint64_t>(float_key(f)) << 32) | static_cast<uint64_t>(~cd[u].y);
      }
    }
  }
  if (nan_seen) report(a.status, SPATTEN_E_NONFINITE);
  __syncthreads();
  const uint32_t m = min(n_bc, static_cast<uint32_t>(kBinCap));
  const uint32_t need = k - above_s;   // 1 <= need <= m
  // T = the need-th largest composite; the selected ones of the sub-bin are counted per chunk
  uint64_t T;
  if (m <= static_cast<uint32_t>(kRThreads)) {   // uniform: sort the sub-bin
    uint64_t x = tid < static_cast<int>(m) ? bc[tid] : 0ull;   // 0: below every composite
    x = bitonic_desc_1024(x, bc);
    if (tid == static_cast<int>(need) - 1) t_s = x;
    const bool s = tid < static_cast<int>(min(need, m));
    const uint32_t j = ~static_cast<uint32_t>(x);
    if (s) atomicOr(&mrow[j >> 5], 1u << (j & 31u));
    const uint32_t chunk = s ? j / kChunk : 0xFFFFFFFFu;
    const uint32_t grp = __match_any_sync(0xffffffffu, chunk);
    if (s && lane == __ffs(grp) - 1) atomicAdd(&cnt[chunk], __popc(grp));
    __syncthreads();
    T = t_s;
  } else {
    // two bits per round (the largest T with count(>= T) >= need)
    uint64_t v[kBinCap / kRThreads];
#pragma unroll
    for (int u = 0; u < kBinCap / kRThreads; ++u) {
      const uint32_t i = tid + u * kRThreads;
      v[u] = i < m ? bc[i] : 0ull;
    }
    const int nv = static_cast<int>((m + kRThreads - 1) / kRThreads);   // live registers (uniform)
    T = 0ull;
    int rnd = 0;
#pragma unroll 1
    for (int b = 62; b >= 0; b -= 2, ++rnd) {
      const uint64_t c1 = T | (1ull << b), c2 = T | (2ull << b), c3 = T | (3ull << b);
      uint32_t x = 0u, y = 0u;
#pragma unroll
      for (int u = 0; u < kBinCap / kRThreads; ++u) {
        if (u < nv) {
          x += (v[u] >= c1 ? 1u : 0u) + (v[u] >= c2 ? 0x10000u : 0u);
          y += v[u] >= c3 ? 1u : 0u;
        }
      }
      x = __reduce_add_sync(0xffffffffu, x);
      y = __reduce_add_sync(0xffffffffu, y);
      if (lane == 0) {
        red[rnd & 1][0][warp] = x;
        red[rnd & 1][1][warp] = y;
      }
      __syncthreads();
      x = __reduce_add_sync(0xffffffffu, red[rnd & 1][0][lane]);
      y = __reduce_add_sync(0xffffffffu, red[rnd & 1][1][lane]);
      T |= static_cast<uint64_t>(((x & 0xFFFFu) >= need) + ((x >> 16) >= need) + (y >= need)) << b;
    }
#pragma unroll
    for (int u = 0; u < kBinCap / kRThreads; ++u) {
      const bool s = u < nv && v[u] >= T && v[u] != 0ull;
      const uint32_t j = ~static_cast<uint32_t>(v[u]);
      if (s) atomicOr(&mrow[j >> 5], 1u << (j & 31u));
      const uint32_t chunk = s ? j / kChunk : 0xFFFFFFFFu;
      const uint32_t grp = __match_any_sync(0xffffffffu, chunk);
      if (s && lane == __ffs(grp) - 1) atomicAdd(&cnt[chunk], __popc(grp));
    }
  }
  const uint32_t t_key = static_cast<uint32_t>(T >> 32), t_idx = ~static_cast<uint32_t>(T);
  // chunk counts: above the window, plus the candidates of the sub-bins before js (all above T),
  // plus the sub-bin's selected candidates (above); warp w takes chunks w, w + 32, ...
  for (int c = warp; c < nchunk; c += kRThreads / 32) {
    const uint32_t* hc = h + static_cast<int64_t>(c) * kBins;
    uint32_t s = (lane < js ? hc[lane] : 0u) + (lane + 32 < js ? hc[lane + 32] : 0u);
    s = __reduce_add_sync(0xffffffffu, s);
    if (lane == 0 && s) atomicAdd(&cnt[c], s);
  }
  __syncthreads();
  // chunk offsets: exclusive prefix sums of the counts (each thread a run of consecutive chunks)
  const int per = (nchunk + kRThreads - 1) / kRThreads;
  const int c0 = min(tid * per, nchunk), c1 = min(c0 + per, nchunk);
  uint32_t s = 0u;
  for (int c = c0; c < c1; ++c) s += cnt[c];
  uint32_t total;
  uint32_t acc = scan1024(s, part, total);
  for (int c = c0; c < c1; ++c) {
    w.chunk_off[static_cast<int64_t>(r) * nchunk + c] = acc;
    acc += cnt[c];
  }
  if (tid == 0) {
    uint32_t* rr = w.res + static_cast<int64_t>(r) * 4;
    rr[0] = 1u;
    rr[1] = t_key;
    rr[2] = t_idx;
    rr[3] = 0u;   // spare
    w.fallback[r] = 0;
  }
}

// The output step: warp w turns the chunk's selection words 16 w .. 16 w + 15 (keys 512 w ..
// 512 w + 511 of the chunk) into indices, staged in shared memory in index order at the output's
// 16-byte phase; the block then writes the chunk's run of indices with aligned 16-byte stores
// (scalar stores only at the run's two ragged ends).  Its global reads (the threshold record, the
// words, the chunk's output offset) are independent of one another.
__global__ void __launch_bounds__(kFThreads, 4) topk_output_kernel(TArgs a, StreamWs w) {
  __shared__ __align__(16) uint32_t sel[kChunk / 32];
  __shared__ __align__(16) int32_t stage[kChunk + 4];
  __shared__ uint32_t wc[kFWarps];
  const int c = blockIdx.x, r = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t rc = static_cast<int64_t>(r) * w.nchunk + c;
  grid_dep_wait();   // everything below reads the resolve step's results
  const uint32_t valid = w.res[static_cast<int64_t>(r) * 4];
  const uint32_t word = lane < kFKeys ? w.gtmask[rc * (kChunk / 32) + warp * kFKeys + lane] : 0u;
  const uint32_t off = w.chunk_off[rc];
  if (!valid) return;   // uniform: the row is redone by the fallback
  if (lane < kFKeys) sel[warp * kFKeys + lane] = word;
  __syncwarp();
  const uint4* words = reinterpret_cast<const uint4*>(&sel[warp * kFKeys]);   // four words per load
  const uint32_t cw = __reduce_add_sync(0xffffffffu, __popc(word));
  if (lane == 0) wc[warp] = cw;
  __syncthreads();
  const uint32_t total = __reduce_add_sync(0xffffffffu, lane < kFWarps ? wc[lane] : 0u);
  int32_t* out = a.idx_out + static_cast<int64_t>(r) * a.ld_out;
  // the output position off + i goes to stage[ph + i], ph = (off + i) - i mod 4 in words of the
  // destination address, so 16-byte groups of the output are 16-byte groups of the stage
  const uint32_t ph = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(out + off) >> 2) & 3u;
  {
    uint32_t pos = ph + __reduce_add_sync(0xffffffffu, lane < warp ? wc[lane] : 0u);
    const int span = c * kChunk + warp * (32 * kFKeys);
    const uint32_t bit = 1u << lane, lt = bit - 1u;
#pragma unroll
    for (int g = 0; g < kFKeys / 4; ++g) {
      const uint4 v = words[g];
      const uint32_t m4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (m4[u] & bit) stage[pos + __popc(m4[u] & lt)] = span + 32 * (4 * g + u) + lane;
        pos += __popc(m4[u]);
      }
    }
  }
  __syncthreads();
  // never past k (always within, when the counts agree)
  const uint32_t kk = static_cast<uint32_t>(a.k);
  const uint32_t cnt = off >= kk ? 0u : min(total, kk - off);
  const uint32_t end = ph + cnt;
  int32_t* base = out + off - ph;   // 16-byte aligned; written only at [ph, end)
  for (uint32_t v = tid; 4 * v < end; v += kFThreads) {
    const uint32_t p = 4 * v;
    if (p >= ph && p + 4 <= end) {
      reinterpret_cast<int4*>(base)[v] = *reinterpret_cast<const int4*>(&stage[p]);
    } else {
#pragma unroll
      for (uint32_t u = 0; u < 4; ++u)
        if (p + u >= ph && p + u < end) base[p + u] = stage[p + u];
    }
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
  take(static_cast<size_t>(R) * 4);                    // ccount
  take(static_cast<size_t>(R) * 4 * 4);                // ends (16-byte rows)
  take(static_cast<size_t>(R) * nchunk * 4);           // chunk_gt
  take(static_cast<size_t>(R) * nchunk * kBins * 4);   // hist
  take(static_cast<size_t>(R) * nchunk * 4);           // chunk_off
  take(static_cast<size_t>(R) * nchunk * (kChunk / 8)); // gtmask
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
  return n >= kStreamMin && (static_cast<int64_t>(n) + kChunk - 1) / kChunk <= kMaxChunks;
}

size_t topk_workspace_bytes(int R, int n, int k) {
  (void)k;
  return stream_fits(R, n) ? stream_ws_bytes(R, n) : 0;
}

int32_t cluster_launch(const TArgs& a, cudaStream_t st);

// a streaming step launched with programmatic stream serialisation (see grid_dep_wait)
int32_t launch_after_previous(void (*kernel)(TArgs, StreamWs), dim3 grid, int threads, size_t smem, cudaStream_t st,
                              const TArgs& g, const StreamWs& v) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SPT_CUDA(cudaLaunchKernelEx(&cfg, kernel, g, v));
  return launch_status();
}

// the four steps for rows [r0, r0 + rows)
int32_t stream_chain(const TArgs& a, const StreamWs& w, int r0, int rows, cudaStream_t st) {
  TArgs g = a;
  g.scores = a.scores + static_cast<int64_t>(r0) * a.ld;
  g.idx_out = a.idx_out + static_cast<int64_t>(r0) * a.ld_out;
  g.R = rows;
  StreamWs v = w;
  v.ends += static_cast<int64_t>(r0) * 4;
  v.ccount += r0;
  v.chunk_gt += static_cast<int64_t>(r0) * w.nchunk;
  v.hist += static_cast<int64_t>(r0) * w.nchunk * kBins;
  v.chunk_off += static_cast<int64_t>(r0) * w.nchunk;
  v.gtmask += static_cast<int64_t>(r0) * w.nchunk * (kChunk / 32);
  v.res += static_cast<int64_t>(r0) * 4;
  v.fallback += r0;
  v.cand += static_cast<int64_t>(r0) * w.cap;
  if (g.n >= 512 * 1024) topk_sample_kernel<16><<<rows, kRThreads, 0, st>>>(g, v);
  else topk_sample_kernel<8><<<rows, kRThreads, 0, st>>>(g, v);
  SPT_TRY(launch_status());
  SPT_TRY(launch_after_previous(topk_filter_kernel, dim3(w.nchunk, rows), kFThreads, 0, st, g, v));
  SPT_TRY(launch_after_previous(topk_resolve_kernel, dim3(rows), kRThreads,
                                static_cast<size_t>(kBinCap) * 8 + static_cast<size_t>(w.nchunk) * 4, st, g, v));
  return launch_after_previous(topk_output_kernel, dim3(w.nchunk, rows), kFThreads, 0, st, g, v);
}

int32_t topk_stream_launch(const TArgs& a, void* ws, cudaStream_t st) {
  static DeviceOnce once;
  int dev = 0;
  SPT_TRY(once_per_device(once, &dev, [](int) -> int32_t {
    SPT_CUDA(cudaFuncSetAttribute(topk_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kBinCap * 8 + kMaxChunks * 4));
    return SPATTEN_OK;
  }));
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
  w.ccount = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * 4));
  w.ends = reinterpret_cast<float*>(take(static_cast<size_t>(R) * 4 * 4));
  w.chunk_gt = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * w.nchunk * 4));
  w.hist = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * w.nchunk * kBins * 4));
  w.chunk_off = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * w.nchunk * 4));
  w.gtmask = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * w.nchunk * (kChunk / 8)));
  w.res = reinterpret_cast<uint32_t*>(take(static_cast<size_t>(R) * 16));
  w.fallback = reinterpret_cast<int32_t*>(take(static_cast<size_t>(R) * 4));
  w.cand = reinterpret_cast<uint2*>(take(static_cast<size_t>(R) * w.cap * 8));
  SPT_TRY(stream_chain(a, w, 0, R, st));
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
  static DeviceOnce once;
  static bool wide_ok[64] = {false};   // 16-CTA clusters can be scheduled on this device
  int dev = 0;
  SPT_TRY(once_per_device(once, &dev, [](int dev) -> int32_t {
    SPT_CUDA(cudaFuncSetAttribute(topk_cluster_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kResident * 4));
    SPT_CUDA(cudaFuncSetAttribute(topk_cluster_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kResident * 4));
    if (cudaFuncSetAttribute(topk_cluster_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(topk_cluster_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
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
      wide_ok[dev] = cudaOccupancyMaxActiveClusters(&clusters, topk_cluster_kernel<false>, &q) == cudaSuccess && clusters >= 4;
    }
    cudaGetLastError();   // the probe above may leave an error behind
    return SPATTEN_OK;
  }));
  int C = pick_cluster(a.n);
  if (C == 8 && a.n > 8 * kResident && wide_ok[dev]) C = 16;
  const int chunk = static_cast<int>((ceil_div(a.n, C) + 3) & ~int64_t(3));
  const size_t smem = static_cast<size_t>(std::min(chunk, kResident)) * 4;
  cudaLaunchConfig_t cfg = {};
  // rows left to the fallback (only_rows) are rare: a few clusters loop over all rows and skip the
  // others, instead of one cluster per row
  cfg.gridDim = dim3(C, a.only_rows ? std::min(a.R, 8) : a.R, 1);
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
  if (a.only_rows) SPT_CUDA(cudaLaunchKernelEx(&cfg, topk_cluster_kernel<true>, a));
  else SPT_CUDA(cudaLaunchKernelEx(&cfg, topk_cluster_kernel<false>, a));
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
  spt::AbiRange nvtx_range("spatten_topk_select");
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
