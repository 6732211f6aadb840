// K1: progressive 12-bit K/V quantization into an int8 MSB plane and a packed 4-bit LSB plane.
//
// SpAtten §III.A "Progressive Quantization" stores K/V so that the MSBs can be fetched alone and
// the LSBs only when a row's attention is too flat; §IV "Quantization Support" splits the fetched
// bits and concatenates MSBs with LSBs.  Codes: q = clamp(rint(float32(x*gain) / s), +-2047),
// MSB = q >> 4, LSB = q & 15, s = amax / 2047 per (sequence, head) block.
//
// Amax mode, small blocks (at most 4096 chunks of 8 elements for bf16, 2048 for float32, e.g.
// 512 rows of 64): one CTA per (b, h) block (gridDim.z selects K or V when both are quantized in
// one launch) holds the block's raw 16-byte words in registers, reduces the amax and writes the
// codes from the same registers: one read.
// Amax mode, larger blocks: one thread-block cluster per (b, h) block; each CTA reduces the amax of
// its rows, the cluster exchanges the partial maxima through distributed shared memory, and every
// CTA then quantizes its rows (a second read that hits L2).  Each thread keeps four 16-byte loads
// in flight.  No scratch memory is needed in either mode.
// Fixed-scale mode (decode append): one thread per 8-element chunk, saturations counted.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace spt {

constexpr int kQThreads = 256;
constexpr int kQBatch = 4;   // 16-byte chunks in flight per thread
constexpr float kQMax = 2047.0f;

struct QTensor {
  const void* x;
  const float* gain;
  int8_t* msb;
  uint8_t* lsb;
  float* scale_out;
  const float* scale_in;
};

struct QArgs {
  QTensor t[2];
  int B, H, n, d_h;
  int64_t ld_tok;
  int64_t ld_gain;
  int cap, row0;
  int32_t* sat;
};

namespace {

// rint(float32(v / s)) without a division per element: t = v * (1/s) (reciprocal correctly
// rounded) lies within 1.5 ulp(t) of the float32 quotient, i.e. within 2^-10 for |t| < 4096, so
// unless t is within 2^-9 of a half-integer both round to the same integer; those rare near-ties
// are recomputed with the IEEE division.  The rounding itself is an add of 1.5 * 2^23, which
// leaves rint(t) (ties to even) in the low mantissa bits; |t| >= 4096 saturates either way and
// returns +-4096.
__device__ __forceinline__ int code_of(float v, float s, float rcp) {
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  const float t = v * rcp;
  if (!(fabsf(t) < 4096.0f)) return t > 0.0f ? 4096 : -4096;
  float tm = t + kMagic;
  if (fabsf(t - (tm - kMagic)) > 0.5f - 0.001953125f) tm = __fdiv_rn(v, s) + kMagic;
  return __float_as_int(tm) - 0x4B400000;
}

// quantize 8 values with scale s (rcp = 1/s, correctly rounded); returns the number of saturated
// codes
__device__ __forceinline__ int quant8(const float* v, float s, float rcp, int8_t* msb_dst, uint8_t* lsb_dst) {
  int sat = 0;
  uint32_t m[2] = {0u, 0u};
  uint32_t l = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int q = code_of(v[i], s, rcp);
    sat += (q > 2047 || q < -2047) ? 1 : 0;
    q = min(max(q, -2047), 2047);
    const int hi = q >> 4;    // arithmetic shift: floor(q / 16)
    const int lo = q & 15;
    m[i >> 2] |= (static_cast<uint32_t>(hi) & 0xFFu) << (8 * (i & 3));
    l |= static_cast<uint32_t>(lo) << (4 * i);
  }
  *reinterpret_cast<uint2*>(msb_dst) = make_uint2(m[0], m[1]);
  *reinterpret_cast<uint32_t*>(lsb_dst) = l;
  return sat;
}

template <typename T>
__device__ __forceinline__ const T* chunk_ptr(const QArgs& a, const QTensor& q, int b, int h, int t, int c) {
  return static_cast<const T*>(q.x) + (static_cast<int64_t>(b) * a.n + t) * a.ld_tok + static_cast<int64_t>(h) * a.d_h + c * 8;
}

__device__ __forceinline__ void apply_gain(const QArgs& a, const QTensor& q, int b, int t, float* v) {
  if (q.gain) {
    const float g = q.gain[static_cast<int64_t>(b) * a.ld_gain + t];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= g;
  }
}

// CT: 16-byte chunks per head row when known at compile time (d_h / 8), 0 otherwise
template <typename T, int CT>
__global__ void __launch_bounds__(kQThreads) quantize_amax_kernel(QArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int S = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const QTensor& q = a.t[blockIdx.z];
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int C = CT ? CT : a.d_h / 8;
  const int rows_per = (a.n + S - 1) / S;
  const int r0 = min(a.n, rank * rows_per), r1 = min(a.n, r0 + rows_per);
  const int total = (r1 - r0) * C;

  __shared__ float red[kQThreads / 32];
  __shared__ float cta_amax;

  // pass 1: amax, kQBatch chunks (8 values each) in flight per thread
  float amax = 0.0f;
#pragma unroll 1
  for (int e0 = threadIdx.x; e0 < total; e0 += kQBatch * kQThreads) {
    float v[kQBatch][8];
#pragma unroll
    for (int u = 0; u < kQBatch; ++u) {
      const int e = e0 + u * kQThreads;
      if (e < total) load8(chunk_ptr<T>(a, q, b, h, r0 + e / C, e % C), v[u]);
    }
#pragma unroll
    for (int u = 0; u < kQBatch; ++u) {
      const int e = e0 + u * kQThreads;
      if (e < total) {
        apply_gain(a, q, b, r0 + e / C, v[u]);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[u][i]));
      }
    }
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
    for (int w = 0; w < kQThreads / 32; ++w) m = fmaxf(m, red[w]);
    cta_amax = m;
  }
  cluster.sync();
  float block_amax = 0.0f;
  for (int r = 0; r < S; ++r) block_amax = fmaxf(block_amax, *cluster.map_shared_rank(&cta_amax, r));
  cluster.sync();   // no CTA leaves while a peer may still read its shared memory

  const float s = block_amax == 0.0f ? 1.0f : __fdiv_rn(block_amax, kQMax);
  const float rcp = __frcp_rn(s);
  if (rank == 0 && threadIdx.x == 0) q.scale_out[bh] = s;

  // pass 2: codes (the rows are read again; they are in L2)
#pragma unroll 1
  for (int e0 = threadIdx.x; e0 < total; e0 += kQBatch * kQThreads) {
    float v[kQBatch][8];
#pragma unroll
    for (int u = 0; u < kQBatch; ++u) {
      const int e = e0 + u * kQThreads;
      if (e < total) load8(chunk_ptr<T>(a, q, b, h, r0 + e / C, e % C), v[u]);
    }
#pragma unroll
    for (int u = 0; u < kQBatch; ++u) {
      const int e = e0 + u * kQThreads;
      if (e < total) {
        const int t = r0 + e / C, c = e % C;
        apply_gain(a, q, b, t, v[u]);
        const int64_t row = static_cast<int64_t>(bh) * a.cap + a.row0 + t;
        quant8(v[u], s, rcp, q.msb + row * a.d_h + c * 8, q.lsb + row * (a.d_h / 2) + c * 4);
      }
    }
  }
}

// eight consecutive elements of a head row kept as raw 16-byte words (one for bf16, two for float)
template <typename T>
struct Chunk8;

template <>
struct Chunk8<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { w = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void get(float* f) const {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // bf16 -> float: the 16 bits become the high half of the word
      f[2 * i] = __uint_as_float(u[i] << 16);
      f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
  }
};

template <>
struct Chunk8<float> {
  uint4 w0, w1;
  __device__ __forceinline__ void load(const float* p) {
    w0 = __ldg(reinterpret_cast<const uint4*>(p));
    w1 = __ldg(reinterpret_cast<const uint4*>(p + 4));
  }
  __device__ __forceinline__ void get(float* f) const {
    f[0] = __uint_as_float(w0.x); f[1] = __uint_as_float(w0.y); f[2] = __uint_as_float(w0.z); f[3] = __uint_as_float(w0.w);
    f[4] = __uint_as_float(w1.x); f[5] = __uint_as_float(w1.y); f[6] = __uint_as_float(w1.z); f[7] = __uint_as_float(w1.w);
  }
};

constexpr int kQBThreads = 512;
template <typename T>
constexpr int block_chunks() { return sizeof(T) == 2 ? 8 : 4; }   // chunks per thread (registers)

// Amax of one bf16 chunk times |gain|: the sign-cleared bit patterns of finite bf16 values order
// like their magnitudes, two patterns per 32-bit unsigned max; multiplying the largest magnitude by
// |gain| rounds like the largest of the rounded products (rounding is monotone).  *nf is set when
// the chunk holds an infinity or a NaN.
__device__ __forceinline__ float chunk_amax_bf16(const uint4 w, float gabs, bool* nf) {
  const uint32_t m2 = __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu), __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu));
  const uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  *nf = *nf || m >= 0x7F80u;
  return __uint_as_float(m << 16) * gabs;
}

// quant8 for a finite amax-mode block (|v| <= amax, so every code is within +-2047 and none
// saturates), on value pairs: t = v * (1/s) and the 1.5 * 2^23 rounding add as paired float
// operations, the near-tie recheck (the IEEE division) only for the rare pair that needs it.  The
// rounded float's bit pattern is 0x4B400000 + q: its bits 4..11 are the MSB byte q >> 4, its
// bits 0..3 the LSB q & 15.
__device__ __forceinline__ void quant8_bf16_finite(const uint4 w, float g, float s, float rcp, int8_t* msb_dst,
                                                   uint8_t* lsb_dst) {
  constexpr float kMagic = 12582912.0f;
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  uint32_t bits[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 v = make_float2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xFFFF0000u));
    v = __fmul2_rn(v, make_float2(g, g));
    const float2 t = __fmul2_rn(v, make_float2(rcp, rcp));
    float2 tm = __fadd2_rn(t, make_float2(kMagic, kMagic));
    const float2 r = __fadd2_rn(tm, make_float2(-kMagic, -kMagic));
    const float2 d = __ffma2_rn(r, make_float2(-1.0f, -1.0f), t);   // t - rint(t), exact
    if (fabsf(d.x) > 0.5f - 0.001953125f) tm.x = __fdiv_rn(v.x, s) + kMagic;
    if (fabsf(d.y) > 0.5f - 0.001953125f) tm.y = __fdiv_rn(v.y, s) + kMagic;
    bits[2 * i] = __float_as_uint(tm.x);
    bits[2 * i + 1] = __float_as_uint(tm.y);
  }
  uint32_t m[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t* b = bits + 4 * h;
    m[h] = __byte_perm(__byte_perm(b[0] >> 4, b[1] >> 4, 0x0040), __byte_perm(b[2] >> 4, b[3] >> 4, 0x0040), 0x5410);
  }
  uint32_t l = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) l |= (bits[i] & 15u) << (4 * i);
  *reinterpret_cast<uint2*>(msb_dst) = make_uint2(m[0], m[1]);
  *reinterpret_cast<uint32_t*>(lsb_dst) = l;
}

// C: chunks per head row (d_h / 8)
template <typename T, int C>
__global__ void __launch_bounds__(kQBThreads) quantize_amax_block_kernel(QArgs a) {
  constexpr int CH = block_chunks<T>();
  constexpr bool kBf = sizeof(T) == 2;
  const QTensor& q = a.t[blockIdx.z];
  const int bh = blockIdx.x;
  const int b = bh / a.H, h = bh % a.H;
  const int total = a.n * C;
  __shared__ float red[kQBThreads / 32];
  Chunk8<T> ch[CH];
#pragma unroll
  for (int u = 0; u < CH; ++u) {
    const int e = threadIdx.x + u * kQBThreads;
    if (e < total) ch[u].load(chunk_ptr<T>(a, q, b, h, e / C, e % C));
  }
  auto gain_of = [&](int e) -> float {
    return q.gain ? q.gain[static_cast<int64_t>(b) * a.ld_gain + e / C] : 1.0f;
  };
  float amax = 0.0f;
  bool nonfinite = false;
#pragma unroll
  for (int u = 0; u < CH; ++u) {
    const int e = threadIdx.x + u * kQBThreads;
    if (e < total) {
      if constexpr (kBf) {
        amax = fmaxf(amax, chunk_amax_bf16(ch[u].w, fabsf(gain_of(e)), &nonfinite));
      } else {
        float v[8];
        ch[u].get(v);
        apply_gain(a, q, b, e / C, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    }
  }
  if (kBf && __syncthreads_or(nonfinite ? 1 : 0)) {
    // an infinity or NaN in the block: the element-wise amax (fmaxf passes over NaNs)
    amax = 0.0f;
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      const int e = threadIdx.x + u * kQBThreads;
      if (e < total) {
        float v[8];
        ch[u].get(v);
        apply_gain(a, q, b, e / C, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    }
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float block_amax = 0.0f;
#pragma unroll
  for (int w = 0; w < kQBThreads / 32; ++w) block_amax = fmaxf(block_amax, red[w]);
  const float s = block_amax == 0.0f ? 1.0f : __fdiv_rn(block_amax, kQMax);
  const float rcp = __frcp_rn(s);
  if (threadIdx.x == 0) q.scale_out[bh] = s;
  const bool fast = kBf && block_amax <= 3.0e38f;   // finite (and not NaN): no code saturates
#pragma unroll
  for (int u = 0; u < CH; ++u) {
    const int e = threadIdx.x + u * kQBThreads;
    if (e < total) {
      const int t = e / C, c = e % C;
      const int64_t row = static_cast<int64_t>(bh) * a.cap + a.row0 + t;
      if constexpr (kBf) {
        if (fast) {
          quant8_bf16_finite(ch[u].w, gain_of(e), s, rcp, q.msb + row * a.d_h + c * 8, q.lsb + row * (a.d_h / 2) + c * 4);
          continue;
        }
      }
      float v[8];
      ch[u].get(v);
      apply_gain(a, q, b, t, v);
      quant8(v, s, rcp, q.msb + row * a.d_h + c * 8, q.lsb + row * (a.d_h / 2) + c * 4);
    }
  }
}

template <typename T, int CT>
__global__ void __launch_bounds__(kQThreads) quantize_fixed_kernel(QArgs a) {
  const QTensor& q = a.t[blockIdx.z];
  const int C = CT ? CT : a.d_h / 8;
  const int64_t total = static_cast<int64_t>(a.B) * a.H * a.n * C;
  int sat = 0;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(kQThreads) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * kQThreads) {
    const int c = static_cast<int>(e % C);
    const int64_t r = e / C;                     // (b*H + h)*n + t
    const int t = static_cast<int>(r % a.n);
    const int bh = static_cast<int>(r / a.n);
    const int b = bh / a.H, h = bh % a.H;
    float v[8];
    load8(chunk_ptr<T>(a, q, b, h, t, c), v);
    apply_gain(a, q, b, t, v);
    const float s = q.scale_in[bh];
    const int64_t row = static_cast<int64_t>(bh) * a.cap + a.row0 + t;
    sat += quant8(v, s, __frcp_rn(s), q.msb + row * a.d_h + c * 8, q.lsb + row * (a.d_h / 2) + c * 4);
  }
  sat = warp_sum_int(sat);
  if (a.sat && (threadIdx.x & 31) == 0 && sat) atomicAdd(a.sat, sat);
}

}  // namespace

// Quantize `ntensors` (1 or 2) tensors of the same shape in one launch.  Either every tensor has
// scale_in (fixed-scale mode) or none has.
int32_t quantize_launch(const QArgs& a, int ntensors, int dtype, cudaStream_t st) {
  if (a.t[0].scale_in) {
    const int64_t chunks = static_cast<int64_t>(a.B) * a.H * a.n * (a.d_h / 8);
    int grid = static_cast<int>(std::min<int64_t>(ceil_div(chunks, kQThreads), 8LL * sm_count()));
    dim3 g(grid, 1, ntensors);
    const bool bf = dtype == SPATTEN_BF16;
    if (a.d_h == 64) {
      if (bf) quantize_fixed_kernel<__nv_bfloat16, 8><<<g, kQThreads, 0, st>>>(a);
      else quantize_fixed_kernel<float, 8><<<g, kQThreads, 0, st>>>(a);
    } else if (a.d_h == 128) {
      if (bf) quantize_fixed_kernel<__nv_bfloat16, 16><<<g, kQThreads, 0, st>>>(a);
      else quantize_fixed_kernel<float, 16><<<g, kQThreads, 0, st>>>(a);
    } else {
      if (bf) quantize_fixed_kernel<__nv_bfloat16, 0><<<g, kQThreads, 0, st>>>(a);
      else quantize_fixed_kernel<float, 0><<<g, kQThreads, 0, st>>>(a);
    }
    return launch_status();
  }
  const int blocks = a.B * a.H;
  const bool bf = dtype == SPATTEN_BF16;
  const int64_t chunks = static_cast<int64_t>(a.n) * (a.d_h / 8);
  if ((a.d_h == 64 || a.d_h == 128) &&
      chunks <= static_cast<int64_t>(kQBThreads) * (bf ? block_chunks<__nv_bfloat16>() : block_chunks<float>())) {
    const dim3 g(blocks, 1, ntensors);
    if (a.d_h == 64) {
      if (bf) quantize_amax_block_kernel<__nv_bfloat16, 8><<<g, kQBThreads, 0, st>>>(a);
      else quantize_amax_block_kernel<float, 8><<<g, kQBThreads, 0, st>>>(a);
    } else {
      if (bf) quantize_amax_block_kernel<__nv_bfloat16, 16><<<g, kQBThreads, 0, st>>>(a);
      else quantize_amax_block_kernel<float, 16><<<g, kQBThreads, 0, st>>>(a);
    }
    return launch_status();
  }
  // enough CTAs for eight per SM (every SM then keeps 2048 threads' loads in flight); at most 8
  // per block (portable cluster size)
  int S = static_cast<int>(ceil_div(8LL * sm_count(), static_cast<int64_t>(blocks) * ntensors));
  S = std::max(1, std::min(S, 8));
  S = std::min<int>(S, std::max(1, a.n / 16));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, blocks, ntensors);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (a.d_h == 64)
    e = bf ? cudaLaunchKernelEx(&cfg, quantize_amax_kernel<__nv_bfloat16, 8>, a)
           : cudaLaunchKernelEx(&cfg, quantize_amax_kernel<float, 8>, a);
  else if (a.d_h == 128)
    e = bf ? cudaLaunchKernelEx(&cfg, quantize_amax_kernel<__nv_bfloat16, 16>, a)
           : cudaLaunchKernelEx(&cfg, quantize_amax_kernel<float, 16>, a);
  else
    e = bf ? cudaLaunchKernelEx(&cfg, quantize_amax_kernel<__nv_bfloat16, 0>, a)
           : cudaLaunchKernelEx(&cfg, quantize_amax_kernel<float, 0>, a);
  if (e != cudaSuccess) {
    record_cuda_error(e);
    return SPATTEN_E_CUDA;
  }
  return launch_status();
}

int32_t quantize_check(const void* x, int32_t dtype, int32_t B, int32_t H, int32_t n, int32_t d_h, int64_t ld_tok,
                       const float* row_gain, int64_t ld_gain, const float* scale_in, const int8_t* msb,
                       const uint8_t* lsb, int32_t cap, int32_t row0, const float* scale_out) {
  if (!x || !msb || !lsb) return SPATTEN_E_ARG;
  if (dtype != SPATTEN_F32 && dtype != SPATTEN_BF16) return SPATTEN_E_ARG;
  if (B < 1 || H < 1 || n < 1 || d_h < 8 || (d_h % 8) != 0) return SPATTEN_E_ARG;
  if (B > 65535 / 1 || static_cast<int64_t>(B) * H > 65535) return SPATTEN_E_ARG;
  if (!scale_in && !scale_out) return SPATTEN_E_ARG;
  if (row0 < 0 || cap < 1 || static_cast<int64_t>(row0) + n > cap) return SPATTEN_E_SHAPE;
  if (ld_tok < static_cast<int64_t>(H) * d_h) return SPATTEN_E_SHAPE;
  if (row_gain && ld_gain < n) return SPATTEN_E_SHAPE;
  const int esz = dtype == SPATTEN_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld_tok * esz) % 16 != 0 || (static_cast<int64_t>(d_h) * esz) % 16 != 0)
    return SPATTEN_E_ALIGN;
  if (!aligned16(msb) || !aligned16(lsb)) return SPATTEN_E_ALIGN;
  return SPATTEN_OK;
}

// K and V of one projection buffer in one launch (used by the cascade driver)
int32_t quantize_kv_pair(const void* k, const void* v, int32_t dtype, int32_t B, int32_t H, int32_t n, int32_t d_h,
                         int64_t ld_tok, const float* k_gain, int64_t ld_gain, const float* k_scale_in,
                         const float* v_scale_in, int8_t* k_msb, uint8_t* k_lsb, int8_t* v_msb, uint8_t* v_lsb,
                         int32_t cap, int32_t row0, float* k_scale_out, float* v_scale_out, int32_t* sat_count,
                         cudaStream_t st) {
  SPT_TRY(quantize_check(k, dtype, B, H, n, d_h, ld_tok, k_gain, ld_gain, k_scale_in, k_msb, k_lsb, cap, row0,
                         k_scale_out));
  SPT_TRY(quantize_check(v, dtype, B, H, n, d_h, ld_tok, nullptr, 0, v_scale_in, v_msb, v_lsb, cap, row0,
                         v_scale_out));
  if ((k_scale_in == nullptr) != (v_scale_in == nullptr)) return SPATTEN_E_ARG;
  QArgs a{};
  a.t[0] = QTensor{k, k_gain, k_msb, k_lsb, k_scale_out, k_scale_in};
  a.t[1] = QTensor{v, nullptr, v_msb, v_lsb, v_scale_out, v_scale_in};
  a.B = B; a.H = H; a.n = n; a.d_h = d_h; a.ld_tok = ld_tok; a.ld_gain = ld_gain; a.cap = cap; a.row0 = row0;
  a.sat = sat_count;
  return quantize_launch(a, 2, dtype, st);
}

}  // namespace spt

extern "C" int32_t spatten_quantize_kv(const void* x, int32_t dtype, int32_t B, int32_t H, int32_t n,
                                       int32_t d_h, int64_t ld_tok, const float* row_gain, int64_t ld_gain,
                                       const float* scale_in, int8_t* msb, uint8_t* lsb, int32_t cap,
                                       int32_t row0, float* scale_out, int32_t* sat_count, void* stream) {
  spt::AbiRange nvtx_range("spatten_quantize_kv");
  using namespace spt;
  SPT_TRY(quantize_check(x, dtype, B, H, n, d_h, ld_tok, row_gain, ld_gain, scale_in, msb, lsb, cap, row0, scale_out));
  QArgs a{};
  a.t[0] = QTensor{x, row_gain, msb, lsb, scale_out, scale_in};
  a.B = B; a.H = H; a.n = n; a.d_h = d_h; a.ld_tok = ld_tok; a.ld_gain = ld_gain; a.cap = cap; a.row0 = row0;
  a.sat = sat_count;
  return quantize_launch(a, 1, dtype, as_stream(stream));
}
