// layernorm.cu -- Z = LayerNorm(Y) over every row of Y, in place.
//
// "1bit量化" (blog.zerodtree.com), knowledge-distillation section: the OneBit
// layer's output Y is followed by Z = LayerNorm(Y).  Per token (a row of Y), over
// its N features: z = (y - mean) / sqrt(var + eps), var the biased variance, no
// affine parameters (the page shows none).
//
// A token's N outputs come from many CTAs of the GEMM, so normalisation is a second
// pass.  bf16 rows of up to 16384 features are read once into registers and written once;
// other rows are read twice (the second read hits L1/L2) and written once.
// One CTA per row.  Statistics: each thread sums y - y0 and (y - y0)^2 in fp32 over
// its strided elements (y0 = the row's first element, so a large mean does not
// cancel the variance away), the CTA combines the partial sums in fp64.
#include <cuda_bf16.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kLnThreads = 256;

__device__ __forceinline__ float bf16_to_f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

template <bool kBF16>
__device__ __forceinline__ float load_y(const void* row, int64_t j) {
  if constexpr (kBF16)
    return bf16_to_f(static_cast<const uint16_t*>(row)[j]);
  else
    return static_cast<const float*>(row)[j];
}

template <bool kBF16>
__device__ __forceinline__ void store_z(void* row, int64_t j, float z) {
  if constexpr (kBF16)
    static_cast<__nv_bfloat16*>(row)[j] = __float2bfloat16_rn(z);
  else
    static_cast<float*>(row)[j] = z;
}

// Sums of two doubles over the CTA in one reduction; every thread gets the results.
__device__ __forceinline__ double2 block_sum2(double a, double b, double2* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = make_double2(a, b);
  __syncthreads();
  double2 t = make_double2(0.0, 0.0);
#pragma unroll
  for (int w = 0; w < kLnThreads / 32; ++w) {
    t.x += red[w].x;
    t.y += red[w].y;
  }
  return t;
}

// Sum of a double over the CTA; every thread gets the result.
__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red is reused between calls
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < kLnThreads / 32; ++w) t += red[w];
  return t;
}

template <bool kBF16>
__global__ void __launch_bounds__(kLnThreads) layernorm_rows_kernel(void* Y, int64_t N, int64_t ld, float eps) {
  __shared__ double red[kLnThreads / 32];
  pdl_wait();  // Y is written by the previous grid
  pdl_launch_dependents();
  const int64_t esz = kBF16 ? 2 : 4;
  void* row = static_cast<char*>(Y) + (int64_t)blockIdx.x * ld * esz;
  const float y0 = load_y<kBF16>(row, 0);
  // 16-byte loads when the row allows them.
  const bool vec = kBF16 && (N % 8 == 0) && ((reinterpret_cast<uintptr_t>(row) & 15) == 0);
  float s1 = 0.f, s2 = 0.f;
  if (vec) {
    const uint4* r4 = static_cast<const uint4*>(row);
    for (int64_t i = threadIdx.x; i < N / 8; i += kLnThreads) {
      const uint4 v = r4[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(w[e] << 16) - y0, hi = __uint_as_float(w[e] & 0xFFFF0000u) - y0;
        s1 += lo + hi;
        s2 = fmaf(lo, lo, fmaf(hi, hi, s2));
      }
    }
  } else {
    for (int64_t j = threadIdx.x; j < N; j += kLnThreads) {
      const float d = load_y<kBF16>(row, j) - y0;
      s1 += d;
      s2 = fmaf(d, d, s2);
    }
  }
  const double S1 = block_sum((double)s1, red);
  const double S2 = block_sum((double)s2, red);
  const double dmean = S1 / (double)N;                   // mean - y0
  const double var = fmax(S2 / (double)N - dmean * dmean, 0.0);
  const float mean = (float)((double)y0 + dmean);
  const float rstd = (float)(1.0 / sqrt(var + (double)eps));
  if (vec) {
    uint4* r4 = static_cast<uint4*>(row);
    for (int64_t i = threadIdx.x; i < N / 8; i += kLnThreads) {
      const uint4 v = r4[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = (__uint_as_float(w[e] << 16) - mean) * rstd;
        const float hi = (__uint_as_float(w[e] & 0xFFFF0000u) - mean) * rstd;
        o[e] = pack_bf16x2(lo, hi);
      }
      r4[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    for (int64_t j = threadIdx.x; j < N; j += kLnThreads)
      store_z<kBF16>(row, j, (load_y<kBF16>(row, j) - mean) * rstd);
  }
}

// bf16 rows with N % 8 == 0, 16-byte aligned, and N / 8 <= 256 V: one pass.  Each thread
// keeps its V 16-byte pieces of the row in registers, so Y is read once and written once.
template <int V>
__global__ void __launch_bounds__(kLnThreads) layernorm_rows_reg_kernel(void* Y, int64_t N, int64_t ld, float eps) {
  __shared__ double2 red[kLnThreads / 32];
  pdl_wait();  // Y is written by the previous grid
  pdl_launch_dependents();
  uint4* r4 = reinterpret_cast<uint4*>(static_cast<char*>(Y) + (int64_t)blockIdx.x * ld * 2);
  const int64_t n8 = N / 8;
  const float y0 = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(r4)[0] << 16);
  uint4 v[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int64_t idx = threadIdx.x + (int64_t)i * kLnThreads;
    v[i] = idx < n8 ? r4[idx] : make_uint4(0u, 0u, 0u, 0u);
  }
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    if (threadIdx.x + (int64_t)i * kLnThreads >= n8) continue;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(w[e] << 16) - y0, hi = __uint_as_float(w[e] & 0xFFFF0000u) - y0;
      s1 += lo + hi;
      s2 = fmaf(lo, lo, fmaf(hi, hi, s2));
    }
  }
  const double2 S = block_sum2((double)s1, (double)s2, red);
  const double S1 = S.x, S2 = S.y;
  const double dmean = S1 / (double)N;  // mean - y0
  const double var = fmax(S2 / (double)N - dmean * dmean, 0.0);
  const float mean = (float)((double)y0 + dmean);
  const float rstd = (float)(1.0 / sqrt(var + (double)eps));
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int64_t idx = threadIdx.x + (int64_t)i * kLnThreads;
    if (idx >= n8) continue;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = (__uint_as_float(w[e] << 16) - mean) * rstd;
      const float hi = (__uint_as_float(w[e] & 0xFFFF0000u) - mean) * rstd;
      o[e] = pack_bf16x2(lo, hi);
    }
    r4[idx] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_layernorm_rows(void* Y, int64_t M, int64_t N, int64_t ld, int y_dtype, float eps,
                                  const LaunchCtx& c) {
  if (M == 0 || N == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)M, 1, 1);
  cfg.blockDim = dim3(kLnThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.pdl ? 1 : 0;
  // bf16 rows that fit 8 pieces of 16 bytes per thread (N <= 16384) and allow 16-byte access
  // take the one-pass kernel.
  const bool reg = y_dtype == OB_OUT_BF16 && N % 8 == 0 && ld % 8 == 0 &&
                   (reinterpret_cast<uintptr_t>(Y) & 15) == 0 && N / 8 <= 8 * kLnThreads;
  const int64_t per = (N / 8 + kLnThreads - 1) / kLnThreads;  // 16-byte pieces per thread
  cudaError_t e;
  if (reg)
    e = per <= 1   ? cudaLaunchKernelEx(&cfg, layernorm_rows_reg_kernel<1>, Y, N, ld, eps)
        : per <= 2 ? cudaLaunchKernelEx(&cfg, layernorm_rows_reg_kernel<2>, Y, N, ld, eps)
        : per <= 4 ? cudaLaunchKernelEx(&cfg, layernorm_rows_reg_kernel<4>, Y, N, ld, eps)
                   : cudaLaunchKernelEx(&cfg, layernorm_rows_reg_kernel<8>, Y, N, ld, eps);
  else
    e = y_dtype == OB_OUT_F32 ? cudaLaunchKernelEx(&cfg, layernorm_rows_kernel<false>, Y, N, ld, eps)
                              : cudaLaunchKernelEx(&cfg, layernorm_rows_kernel<true>, Y, N, ld, eps);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ob
