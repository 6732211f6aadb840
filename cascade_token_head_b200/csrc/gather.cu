// K5: gather of kept rows (token rows of X, importance entries, head blocks) by an index list,
// with optional index-map composition.
//
// SpAtten §III.A "Cascade Token Pruning": a pruned token's Q, K and V leave every following head
// and layer; §IV "Architecture Overview": pruning makes row access random, so the accelerator
// routes random addresses across all HBM channels; §IV.B "Zero Elimination" compacts the
// survivors.  On B200 the equivalent is one warp per kept row issuing coalesced 16-byte copies,
// which keeps every request a full 32-byte sector regardless of which rows survive.
#include "common.cuh"

namespace spt {
namespace {

constexpr int kGThreads = 256;
constexpr int kRowsPerCta = kGThreads / 32;

struct GArgs {
  const char* src;
  int64_t src_batch, src_row;
  int n_src;
  int64_t row_bytes;
  int R;
  const int32_t* idx;
  int64_t ld_idx;
  int k;
  char* dst;
  int64_t dst_batch, dst_row;
  const int32_t* comp_in;
  int64_t ld_comp;
  int32_t* comp_out;
  int check;
  int32_t* status;
};

template <int VEC>
__global__ void __launch_bounds__(kGThreads) gather_rows_kernel(GArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y;
  const int j = blockIdx.x * kRowsPerCta + warp;
  if (j >= a.k) return;
  const int32_t i = a.idx[static_cast<int64_t>(r) * a.ld_idx + j];
  if (a.check && (i < 0 || i >= a.n_src)) {
    if (lane == 0) report(a.status, SPATTEN_E_INDEX);
    return;
  }
  if (a.comp_out && lane == 0)
    a.comp_out[static_cast<int64_t>(r) * a.ld_idx + j] = a.comp_in[static_cast<int64_t>(r) * a.ld_comp + i];
  const char* s = a.src + r * a.src_batch + static_cast<int64_t>(i) * a.src_row;
  char* d = a.dst + r * a.dst_batch + static_cast<int64_t>(j) * a.dst_row;
  if (VEC == 16) {
    // four 16-byte loads in flight per lane before the stores
    const int64_t nv = a.row_bytes / 16;
    const uint4* s4 = reinterpret_cast<const uint4*>(s);
    uint4* d4 = reinterpret_cast<uint4*>(d);
    for (int64_t c0 = lane; c0 < nv; c0 += 128) {
      uint4 r4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < nv) r4[u] = __ldg(s4 + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < nv) d4[c0 + 32 * u] = r4[u];
    }
  } else {
    const int64_t nv = a.row_bytes / 4;
    for (int64_t c = lane; c < nv; c += 32)
      reinterpret_cast<uint32_t*>(d)[c] = __ldg(reinterpret_cast<const uint32_t*>(s) + c);
  }
}

// many short rows (row_bytes <= 16): one thread per row
__global__ void __launch_bounds__(kGThreads) gather_small_kernel(GArgs a) {
  const int r = blockIdx.y;
  const int j = blockIdx.x * kGThreads + threadIdx.x;
  if (j >= a.k) return;
  const int32_t i = a.idx[static_cast<int64_t>(r) * a.ld_idx + j];
  if (a.check && (i < 0 || i >= a.n_src)) {
    report(a.status, SPATTEN_E_INDEX);
    return;
  }
  if (a.comp_out)
    a.comp_out[static_cast<int64_t>(r) * a.ld_idx + j] = a.comp_in[static_cast<int64_t>(r) * a.ld_comp + i];
  const uint32_t* s = reinterpret_cast<const uint32_t*>(a.src + r * a.src_batch + static_cast<int64_t>(i) * a.src_row);
  uint32_t* d = reinterpret_cast<uint32_t*>(a.dst + r * a.dst_batch + static_cast<int64_t>(j) * a.dst_row);
  for (int64_t c = 0; c < a.row_bytes / 4; ++c) d[c] = __ldg(s + c);
}

}  // namespace

int32_t gather_launch(const GArgs& a, cudaStream_t st) {
  if (a.k == 0) return SPATTEN_OK;
  const bool vec16 = (a.row_bytes % 16 == 0) && aligned16(a.src) && aligned16(a.dst) &&
                     a.src_batch % 16 == 0 && a.src_row % 16 == 0 && a.dst_batch % 16 == 0 &&
                     a.dst_row % 16 == 0;
  if (a.row_bytes <= 16) {
    dim3 grid(static_cast<unsigned>(ceil_div(a.k, kGThreads)), a.R);
    gather_small_kernel<<<grid, kGThreads, 0, st>>>(a);
  } else {
    dim3 grid(static_cast<unsigned>(ceil_div(a.k, kRowsPerCta)), a.R);
    if (vec16)
      gather_rows_kernel<16><<<grid, kGThreads, 0, st>>>(a);
    else
      gather_rows_kernel<4><<<grid, kGThreads, 0, st>>>(a);
  }
  return launch_status();
}

}  // namespace spt

extern "C" int32_t spatten_gather_kept(const void* src, int64_t src_batch, int64_t src_row,
                                       int32_t n_src, int64_t row_bytes, int32_t R,
                                       const int32_t* idx, int64_t ld_idx, int32_t k, void* dst,
                                       int64_t dst_batch, int64_t dst_row,
                                       const int32_t* compose_in, int64_t ld_compose,
                                       int32_t* compose_out, int32_t check_index,
                                       int32_t* dev_status, void* stream) {
  spt::AbiRange nvtx_range("spatten_gather_kept");
  using namespace spt;
  if (R < 1 || k < 0 || n_src < 1) return SPATTEN_E_ARG;
  if (k == 0) return SPATTEN_OK;
  if (!src || !dst || !idx) return SPATTEN_E_ARG;
  if (row_bytes <= 0 || row_bytes % 4 != 0) return SPATTEN_E_ARG;
  if (ld_idx < k) return SPATTEN_E_SHAPE;
  if ((compose_in == nullptr) != (compose_out == nullptr)) return SPATTEN_E_ARG;
  if (compose_in && ld_compose < n_src) return SPATTEN_E_SHAPE;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 4 != 0 ||
      src_batch % 4 != 0 || src_row % 4 != 0 || dst_batch % 4 != 0 || dst_row % 4 != 0)
    return SPATTEN_E_ALIGN;
  GArgs a{static_cast<const char*>(src), src_batch, src_row, n_src, row_bytes, R, idx, ld_idx, k,
          static_cast<char*>(dst), dst_batch, dst_row, compose_in, ld_compose, compose_out,
          check_index, dev_status};
  return gather_launch(a, as_stream(stream));
}
