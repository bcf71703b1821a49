// linear_simt.cu -- CUDA-core sign mat-vec: Y = [(X ⊙ b^T) S^T] ⊙ a^T with adds only.
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": X W^T ≈ [(X ⊙ b^T) W_sign^T] ⊙ a^T.
// "Addition is almost all you need ..." (gist.science), "Methodologie": products
// with +/-1 matrices become additions and subtractions.
//
// Each warp owns rows of S; lane l streams 128-bit groups of four packed words
// (group index c = l + 32 j), so a warp load covers 512 contiguous bytes.  The
// pre-scaled activations x' = x ⊙ b live in shared memory as fp32 in a layout
// where lane l always reads bank (const + l): element (token m, bit i, word q of
// group c) sits at ((m*32 + i)*Q + q) * pitch + c.  Sign bit i of a word is
// moved to bit 31 and XORed into x' before the add, so no multiply touches a
// sign.  Lane partial sums are reduced with warp shuffles; the output scale a
// and the store are fused.  Handles MT <= 4 tokens per pass (the host loops
// over token groups); it is the baseline the tensor-core decode kernel is
// measured against.
#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / 32;
constexpr int kRowsPerWarp = 2;
constexpr int kRowsPerCta = kSimtWarps * kRowsPerWarp;
constexpr int kStageFloats = 24576;  // ~96 KB of staged x' per chunk

// Groups (of Q words) staged per chunk so that MT x 32 x Q x pitch floats fit the stage.
template <int MT, int Q>
__host__ __device__ constexpr int groups_per_chunk() { return kStageFloats / (MT * 32 * Q) - 1; }

template <int MT, int Q>
__global__ void __launch_bounds__(kSimtThreads) sign_gemv_simt_kernel(SignGemmArgs g, int64_t m0) {
  extern __shared__ float xs[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t K = g.K;
  const int64_t Wd = K / 32;           // words per row
  const int64_t G = Wd / Q;            // groups per row
  const int64_t mt = min64(MT, g.M - m0);

  float acc[kRowsPerWarp][MT];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

  const int64_t row0 = (int64_t)blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;

  constexpr int kChunk = groups_per_chunk<MT, Q>();
  for (int64_t c0 = 0; c0 < G; c0 += kChunk) {
    const int cg = (int)min64(kChunk, G - c0);
    const int pitch = cg | 1;  // odd pitch: conflict-free staging stores
    __syncthreads();
    // Stage x'[m][k] for k in [32*Q*c0, 32*Q*(c0+cg)).
    const int total = MT * 32 * Q * cg;
    for (int idx = threadIdx.x; idx < total; idx += kSimtThreads) {
      const int m = idx / (32 * Q * cg);
      const int rem = idx - m * (32 * Q * cg);
      const int w_local = rem >> 5;       // word within chunk
      const int i = rem & 31;             // bit
      const int c = w_local / Q, q = w_local - c * Q;
      const int64_t k = (c0 * Q + w_local) * 32 + i;
      float v = 0.f;
      if (m < mt) {
        v = bf16_bits_to_float(g.X[(m0 + m) * K + k]);
        if (g.iscale) v *= __ldg(g.iscale + k);
      }
      xs[((m * 32 + i) * Q + q) * pitch + c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int64_t n = row0 + r;
      if (n >= g.R) break;
      const uint32_t* srow = g.S + n * Wd + c0 * Q;
      for (int c = lane; c < cg; c += 32) {
        uint32_t wq[Q];
        if constexpr (Q == 4) {
          const uint4 v = __ldcs(reinterpret_cast<const uint4*>(srow) + c);
          wq[0] = v.x; wq[1] = v.y; wq[2] = v.z; wq[3] = v.w;
        } else {
          wq[0] = __ldcs(srow + c);
        }
#pragma unroll
        for (int q = 0; q < Q; ++q) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t sbit = (wq[q] << (31 - i)) & 0x80000000u;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const float x = xs[((m * 32 + i) * Q + q) * pitch + c];
              acc[r][m] += __uint_as_float(__float_as_uint(x) ^ sbit);
            }
          }
        }
      }
    }
  }

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
      v *= __ldg(g.oscale + n);
      const int64_t off = (m0 + lane) * g.ldy + n;
      if (g.y_dtype == OB_OUT_F32)
        static_cast<float*>(g.Y)[off] = v;
      else
        static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(v);
    }
  }
}

template <int MT, int Q>
cudaError_t launch_one(const SignGemmArgs& g, int64_t m0, const LaunchCtx& c) {
  const int64_t G = g.K / 32 / Q;
  const int cg = (int)std::min<int64_t>(groups_per_chunk<MT, Q>(), G);
  const size_t smem = sizeof(float) * (size_t)MT * 32 * Q * (size_t)(cg | 1);
  auto kern = sign_gemv_simt_kernel<MT, Q>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const unsigned blocks = (unsigned)((g.R + kRowsPerCta - 1) / kRowsPerCta);
  kern<<<blocks, kSimtThreads, smem, c.stream>>>(g, m0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sign_gemm_simt(const SignGemmArgs& g, const LaunchCtx& c) {
  const bool vec4 = ((g.K / 32) % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.S) & 15) == 0);
  for (int64_t m0 = 0; m0 < g.M; m0 += 4) {
    const int64_t mt = std::min<int64_t>(4, g.M - m0);
    cudaError_t e;
    if (mt == 1)
      e = vec4 ? launch_one<1, 4>(g, m0, c) : launch_one<1, 1>(g, m0, c);
    else if (mt == 2)
      e = vec4 ? launch_one<2, 4>(g, m0, c) : launch_one<2, 1>(g, m0, c);
    else
      e = vec4 ? launch_one<4, 4>(g, m0, c) : launch_one<4, 1>(g, m0, c);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace ob
