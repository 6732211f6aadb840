// Shared device/host helpers of libspatten (sm_100a).  Nothing here is specific to one kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "spatten.h"

namespace spt {

// An NVTX range over one C-ABI call, named after the call: it shows the call's span (host
// enqueue) in profiler timelines; without a profiler attached the push and pop do nothing.
struct AbiRange {
  explicit AbiRange(const char* name) { nvtxRangePushA(name); }
  ~AbiRange() { nvtxRangePop(); }
  AbiRange(const AbiRange&) = delete;
  AbiRange& operator=(const AbiRange&) = delete;
};

// ----------------------------------------------------------------------------------------------
// host-side status helpers
// ----------------------------------------------------------------------------------------------
void record_cuda_error(cudaError_t e);                 // thread-local message for the ABI
int32_t launch_status();                               // cudaGetLastError -> status
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

#define SPT_TRY(expr)                                  \
  do {                                                 \
    int32_t _s = (expr);                               \
    if (_s != SPATTEN_OK) return _s;                   \
  } while (0)

#define SPT_CUDA(expr)                                 \
  do {                                                 \
    cudaError_t _e = (expr);                           \
    if (_e != cudaSuccess) {                           \
      ::spt::record_cuda_error(_e);                    \
      return SPATTEN_E_CUDA;                           \
    }                                                  \
  } while (0)

// Bump allocator over a caller-provided workspace (no device allocation).
struct WsCursor {
  char* base;
  size_t size;
  size_t used = 0;
  WsCursor(void* b, size_t s) : base(static_cast<char*>(b)), size(s) {}
  template <typename T>
  T* take(size_t count) {
    size_t off = align_up(used, 256);
    used = off + count * sizeof(T);
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
  bool fits() const { return used <= size; }
};

// Number of SMs of the current device (cached per device).
int sm_count();

// First-call set-up (kernel attributes, capability probes) once per device ordinal.  The first
// caller on a device runs `setup(dev)` under a lock; callers from other host threads wait for it,
// so no launch can run before its attributes are set.  A set-up that fails is tried again on the
// next call.  Returns the set-up's status (SPATTEN_OK once it has succeeded) and the device in *dev.
struct DeviceOnce {
  std::mutex mu;
  std::atomic<bool> done[64] = {};
};
template <typename F>
int32_t once_per_device(DeviceOnce& once, int* dev_out, F&& setup) {
  int dev = 0;
  SPT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return SPATTEN_E_UNSUPPORTED;
  *dev_out = dev;
  if (once.done[dev].load(std::memory_order_acquire)) return SPATTEN_OK;
  std::lock_guard<std::mutex> lock(once.mu);
  if (once.done[dev].load(std::memory_order_relaxed)) return SPATTEN_OK;
  const int32_t s = setup(dev);
  if (s == SPATTEN_OK) once.done[dev].store(true, std::memory_order_release);
  return s;
}

// ----------------------------------------------------------------------------------------------
// device helpers
// ----------------------------------------------------------------------------------------------
__device__ __forceinline__ void report(int32_t* st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

__device__ __forceinline__ float ld_as_float(const float* p) { return *p; }
__device__ __forceinline__ float ld_as_float(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ void st_from_float(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_from_float(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// 8 consecutive elements -> float[8] (16-byte or 32-byte aligned vector load)
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float* f) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Order-preserving map float -> uint32 (larger float -> larger key); -0.0 maps like +0.0 (adding
// +0.0 turns -0.0 into +0.0 and leaves every other non-NaN value as it is).  Negative values take
// all bits flipped, the others the sign bit set.
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

}  // namespace spt
