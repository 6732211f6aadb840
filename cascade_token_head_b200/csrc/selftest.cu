// spatten_selftest_exp2_poly: evaluates, element by element, the FMA-pipe 2^x that the
// tensor-core attention kernels use for part of their softmax exponentials, so tests can hold it
// to its error bound against a float64 reference.
#include "common.cuh"
#include "exp2_poly.cuh"

namespace spt {
namespace {

__global__ void __launch_bounds__(256) exp2_poly_kernel(const float* x, float* y, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.0f);
  const float2 out = exp2_poly2(in);
  y[i] = out.x;
  if (i + 1 < n) y[i + 1] = out.y;
}

}  // namespace
}  // namespace spt

extern "C" int32_t spatten_selftest_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  spt::AbiRange nvtx_range("spatten_selftest_exp2_poly");
  if (!x || !y || n < 1) return SPATTEN_E_ARG;
  const int64_t pairs = (n + 1) / 2;
  const int64_t blocks = (pairs + 255) / 256;
  if (blocks > 0x7FFFFFFF) return SPATTEN_E_ARG;
  spt::exp2_poly_kernel<<<static_cast<unsigned>(blocks), 256, 0, spt::as_stream(stream)>>>(x, y, n);
  return spt::launch_status();
}
