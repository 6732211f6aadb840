// Status strings, CUDA error capture and device queries of the C ABI.
#include <atomic>
#include <cstdio>
#include <cstring>

#include "attention.cuh"
#include "common.cuh"

namespace spt {

static thread_local char g_last_cuda_error[256] = "no CUDA error recorded";
static std::atomic<uint64_t> g_launches{0};

void record_cuda_error(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
}

int32_t launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return SPATTEN_E_CUDA;
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return SPATTEN_OK;
}

uint64_t launches() { return g_launches.load(std::memory_order_relaxed); }

int sm_count() {
  static std::atomic<int> cached[64] = {};   // every thread that fills an entry writes the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int v = cached[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cached[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

}  // namespace spt

extern "C" int32_t spatten_abi_version(void) { return SPATTEN_ABI_VERSION; }

extern "C" const char* spatten_status_string(int32_t s) {
  switch (s) {
    case SPATTEN_OK: return "SPATTEN_OK";
    case SPATTEN_E_ARG: return "SPATTEN_E_ARG: null pointer or out-of-range argument";
    case SPATTEN_E_SHAPE: return "SPATTEN_E_SHAPE: inconsistent sizes";
    case SPATTEN_E_ALIGN: return "SPATTEN_E_ALIGN: 16-byte alignment required";
    case SPATTEN_E_WORKSPACE: return "SPATTEN_E_WORKSPACE: workspace missing or too small";
    case SPATTEN_E_NONFINITE: return "SPATTEN_E_NONFINITE: NaN input";
    case SPATTEN_E_CUDA: return "SPATTEN_E_CUDA: CUDA error (see spatten_last_cuda_error)";
    case SPATTEN_E_TIMEOUT: return "SPATTEN_E_TIMEOUT: bounded device wait gave up";
    case SPATTEN_E_UNSUPPORTED: return "SPATTEN_E_UNSUPPORTED: configuration not implemented";
    case SPATTEN_E_INDEX: return "SPATTEN_E_INDEX: index list entry out of range";
    case SPATTEN_E_RANGE: return "SPATTEN_E_RANGE: a value outside the range of the kernel's operand type";
    default: return "SPATTEN_E_UNKNOWN";
  }
}

extern "C" const char* spatten_last_cuda_error(void) { return spt::g_last_cuda_error; }

extern "C" uint64_t spatten_kernel_launch_count(void) { return spt::launches(); }

namespace spt {
namespace {
std::atomic<uint32_t> g_wait_limit{0};
}
uint32_t wait_limit_setting() {
  const uint32_t v = g_wait_limit.load(std::memory_order_relaxed);
  return v ? v : kDefaultWaitLimit;
}
}  // namespace spt

extern "C" void spatten_set_wait_limit(uint32_t polls) { spt::g_wait_limit.store(polls, std::memory_order_relaxed); }
