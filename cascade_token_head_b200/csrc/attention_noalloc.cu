// spatten_attention_layer_noalloc: the attention layer for callers that cannot allocate memory.
//
// Some callers of this library have no way to allocate device memory: a plugin inside a host
// application that owns every allocation, a real-time loop that must not enter the CUDA
// allocator, or code that only receives its input and output buffers from someone else.  They
// cannot provide the workspace that spatten_attention_layer asks for.  This entry point runs the
// same attention kernels with their scratch (the per-CTA importance partial sums) placed in a
// fixed array in device global memory that belongs to the library itself.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kScratchBytes of it until the process exits.  Host code cannot use the variable's name as a
// device address, so the first call on each device (with that device current) looks the address
// up with cudaGetSymbolAddress and caches it; that first call should therefore happen before any
// stream capture.  All calls share the one array, so calls that overlap on the GPU (on different
// streams, or from different threads) race on it.  Every byte a call reads from the array is
// written earlier in the same call, so nothing needs clearing between calls.
#include <mutex>

#include "attention.cuh"

namespace spt {
namespace {

constexpr size_t kScratchBytes = SPATTEN_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};   // device address of g_scratch, per device ordinal

int32_t scratch_address(void** out) {
  int dev = 0;
  SPT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return SPATTEN_E_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      record_cuda_error(e);
      return SPATTEN_E_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SPATTEN_OK;
}

}  // namespace
}  // namespace spt

extern "C" int32_t spatten_attention_layer_noalloc(const spatten_attn_args* a, void* stream) {
  spt::AbiRange nvtx_range("spatten_attention_layer_noalloc");
  using namespace spt;
  if (!a) return SPATTEN_E_ARG;
  const size_t need = spatten_attention_workspace_size(a);
  if (need == 0) return attention_layer_timed(a, nullptr, 0, as_stream(stream), nullptr, nullptr);  // reports the argument error
  if (need > kScratchBytes) return SPATTEN_E_WORKSPACE;
  void* scratch = nullptr;
  SPT_TRY(scratch_address(&scratch));
  return attention_layer_timed(a, scratch, kScratchBytes, as_stream(stream), nullptr, nullptr);
}
