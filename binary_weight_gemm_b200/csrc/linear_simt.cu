// linear_simt.cu -- CUDA-core sign mat-vec: Y = [(X ⊙ b^T) S^T] ⊙ a^T with adds only.
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": X W^T ≈ [(X ⊙ b^T) W_sign^T] ⊙ a^T.
// "Addition is almost all you need ..." (gist.science), "Methodologie": products
// with +/-1 matrices become additions and subtractions.
//
// Each warp owns kRowsPerWarp rows of S.  K is processed in chunks of 32 lane
// groups; lane l owns group l of the chunk, i.e. Q consecutive packed words
// loaded with one 128-bit (Q = 4) or 32-bit (Q = 1) load, so a warp load covers
// 512 (or 128) contiguous bytes.  The pre-scaled activations x' = x ⊙ b live in
// shared memory as fp32 in a layout where lane l always reads bank (const + l):
// element (token m, bit i, word q of group c) sits at ((m*32 + i)*Q + q) * 33 + c.
// Sign bit i of a word is moved to bit 31 and XORed into x' before the add, so no
// multiply touches a sign.  Lane partial sums are reduced with warp shuffles; the
// output scale a and the store are fused.  At decode sizes the kernel is
// latency-bound, so every global load of a chunk (the warp's sign words, then
// the activations and scales it stages) is issued before any of them is used.
// Handles MT <= 4 tokens per pass (the host loops over token groups); a single
// token uses the lookup-table variant below.
#include "ob_device.cuh"
#include "ob_internal.h"
#include "lut_block.cuh"

namespace ob {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / 32;
// Rows per warp shrink as tokens per pass grow, to keep the accumulators in registers.
template <int MT>
__host__ __device__ constexpr int rows_per_warp() { return MT >= 4 ? 1 : (MT == 2 ? 2 : 4); }
constexpr int kPitch = 33;  // 32 groups + 1: odd pitch

// Programmatic dependent launch: every read of an input comes after pdl_wait, and
// the next grid is released after it, so at most one grid waits ahead.  (No L2
// prefetch of the weights here: on B200 it made these short kernels slower.)
__device__ __forceinline__ void prologue_wait() {
  pdl_wait();
  pdl_launch_dependents();
}

template <int MT, int Q>
__global__ void __launch_bounds__(kSimtThreads) sign_gemv_simt_kernel(SignGemmArgs g, int64_t m0) {
  constexpr int kRowsPerWarp = rows_per_warp<MT>();
  constexpr int kRowsPerCta = kSimtWarps * kRowsPerWarp;
  extern __shared__ float xs[];  // [MT][32][Q][kPitch]
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t K = g.K;
  const int64_t Wd = K / 32;              // words per row
  const int64_t G = (Wd + Q - 1) / Q;     // groups per row (Q = 4 only when Wd % 4 == 0)
  const int64_t mt = min64(MT, g.M - m0);
  const int64_t row0 = (int64_t)blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
  prologue_wait();

  float acc[kRowsPerWarp][MT];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

  constexpr int kChunkK = 32 * Q * 32;                 // k per chunk: 32 groups of Q words
  constexpr int kPerThread = kChunkK / kSimtThreads;   // staged k per thread (16 or 4)
  for (int64_t c0 = 0; c0 < G; c0 += 32) {
    // 1. This lane's sign words for every row of the warp (independent loads).
    uint32_t wq[kRowsPerWarp][Q];
    const int64_t grp = c0 + lane;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int64_t n = row0 + r;
      const bool ok = n < g.R && grp < G;
      const uint32_t* srow = g.S + (ok ? n : 0) * Wd;
      if constexpr (Q == 4) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ok) v = __ldcs(reinterpret_cast<const uint4*>(srow) + grp);
        wq[r][0] = v.x; wq[r][1] = v.y; wq[r][2] = v.z; wq[r][3] = v.w;
      } else {
        wq[r][0] = ok ? __ldcs(srow + grp) : 0u;
      }
    }
    // 2. Stage x' for this chunk: thread t owns kPerThread consecutive k for all tokens.
    {
      const int64_t kb = c0 * Q * 32 + (int64_t)threadIdx.x * kPerThread;
      float sc[kPerThread];
      uint32_t xv[MT][kPerThread / 2];  // bf16 pairs, as loaded
#pragma unroll
      for (int e = 0; e < kPerThread; e += 4) {
        float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kb + e < K) s4 = g.iscale ? __ldg(reinterpret_cast<const float4*>(g.iscale + kb + e))
                                      : make_float4(1.f, 1.f, 1.f, 1.f);
        sc[e] = s4.x; sc[e + 1] = s4.y; sc[e + 2] = s4.z; sc[e + 3] = s4.w;
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int e = 0; e < kPerThread; e += 4) {
          uint2 v = make_uint2(0u, 0u);
          if (m < mt && kb + e < K) v = __ldg(reinterpret_cast<const uint2*>(g.X + (m0 + m) * K + kb + e));
          xv[m][e / 2] = v.x;
          xv[m][e / 2 + 1] = v.y;
        }
      }
      __syncthreads();  // previous chunk's readers are done with xs
#pragma unroll
      for (int e = 0; e < kPerThread; ++e) {
        const int kl = threadIdx.x * kPerThread + e;  // k within the chunk
        const int w_local = kl >> 5, i = kl & 31;
        const int c = w_local / Q, q = w_local % Q;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint32_t pr = xv[m][e / 2];
          const float x = __uint_as_float((e & 1) ? (pr & 0xFFFF0000u) : (pr << 16));
          xs[((m * 32 + i) * Q + q) * kPitch + c] = x * sc[e];
        }
      }
      __syncthreads();
    }
    // 3. Select/add: sign bit i of each word XORed into x'.
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
#pragma unroll
      for (int q = 0; q < Q; ++q) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t sbit = (wq[r][q] << (31 - i)) & 0x80000000u;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float x = xs[((m * 32 + i) * Q + q) * kPitch + lane];
            acc[r][m] += __uint_as_float(__float_as_uint(x) ^ sbit);
          }
        }
      }
    }
  }

  // 4. Warp reduction, output scale, store.
  float osc[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) osc[r] = (row0 + r < g.R) ? __ldg(g.oscale + row0 + r) : 0.f;
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int64_t n = row0 + r;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float v = acc[r][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r][m] = v;
    }
    if (n < g.R && lane < mt) {
      float v = 0.f;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m == lane) v = acc[r][m];
      v *= osc[r];
      const int64_t off = (m0 + lane) * g.ldy + n;
      if (g.y_dtype == OB_OUT_F32)
        static_cast<float*>(g.Y)[off] = v;
      else
        static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(v);
    }
  }
}

// Single-token kernel: one CTA per 32-row table-lookup block (lut_block.cuh).  With
// static weights (kStatic: the previous grid did not write S or the scales) the first
// chunk's sign words and the output scales are loaded before the programmatic-launch
// wait, so that they stream in while the previous grid finishes.
template <int Q, bool kStatic>
__global__ void __launch_bounds__(kSimtThreads) sign_gemv_lut_kernel(SignGemmArgs g, int64_t m0) {
  extern __shared__ float lut[];
  const int64_t row_base = (int64_t)blockIdx.x * lutb::kRowsPerBlock;
  const int64_t row0 = lutb::warp_row0(row_base);
  uint32_t wq[lutb::kRowsPerWarp][Q];
  float osc[lutb::kRowsPerWarp];
  if constexpr (kStatic) {
    lutb::load_signs<Q>(g, row0, 0, wq, threadIdx.x & 31);
    lutb::load_oscale(g, row0, osc);
  }
  prologue_wait();
  if constexpr (!kStatic) {
    lutb::load_signs<Q>(g, row0, 0, wq, threadIdx.x & 31);
    lutb::load_oscale(g, row0, osc);
  }
  lutb::block<Q, false>(g, m0, row_base, lut, wq, osc);
}

// Launch with programmatic stream serialization when enabled: the kernel may
// start while the previous grid in the stream is still running.
template <typename Kern>
cudaError_t launch_pdl(Kern kern, int64_t blocks, size_t smem, const SignGemmArgs& g, int64_t m0,
                       const LaunchCtx& c) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, 1, 1);
  cfg.blockDim = dim3(kSimtThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, g, m0);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int Q>
cudaError_t launch_lut(const SignGemmArgs& g, int64_t m0, const LaunchCtx& c) {
  const size_t smem = sizeof(float) * 16 * 32 * Q * 8;
  auto kern = g.static_w ? sign_gemv_lut_kernel<Q, true> : sign_gemv_lut_kernel<Q, false>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  constexpr int kRowsPerCta = kSimtWarps * 4;
  return launch_pdl(kern, (g.R + kRowsPerCta - 1) / kRowsPerCta, smem, g, m0, c);
}

template <int MT, int Q>
cudaError_t launch_one(const SignGemmArgs& g, int64_t m0, const LaunchCtx& c) {
  const size_t smem = sizeof(float) * (size_t)MT * 32 * Q * kPitch;
  auto kern = sign_gemv_simt_kernel<MT, Q>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  constexpr int kRowsPerCta = kSimtWarps * rows_per_warp<MT>();
  return launch_pdl(kern, (g.R + kRowsPerCta - 1) / kRowsPerCta, smem, g, m0, c);
}

}  // namespace

cudaError_t launch_sign_gemm_simt(const SignGemmArgs& g, const LaunchCtx& c) {
  const bool vec4 = ((g.K / 32) % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.S) & 15) == 0);
  for (int64_t m0 = 0; m0 < g.M; m0 += 4) {
    const int64_t mt = std::min<int64_t>(4, g.M - m0);
    cudaError_t e;
    if (mt == 1)
      e = vec4 ? launch_lut<4>(g, m0, c) : launch_lut<1>(g, m0, c);
    else if (mt == 2)
      e = vec4 ? launch_one<2, 4>(g, m0, c) : launch_one<2, 1>(g, m0, c);
    else
      e = vec4 ? launch_one<4, 4>(g, m0, c) : launch_one<4, 1>(g, m0, c);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace ob
