// linear_i8.cu -- the one- and two-token sign product on int8 tensor cores
// (i8_block.cuh), one call.
//
//   Y[m, n] = oscale[n] * sum_k (x[m, k] * iscale[k]) * s[n, k],   M <= 2 per pass
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T;
// each of DBF's two sign products ("Addition is almost all you need ...",
// "Methodologie") is one call.
//
// A CTA owns RT = 2 row tiles (32 rows) and all of K, taken in chunks of super-blocks
// (512 k) that fit shared memory.  Per chunk: every warp requests the packed words of its
// items (row tile warp % 2, super-blocks warp / 2, + 4, ...); each warp stages (token,
// super-block) pairs on its own (largest |x'|, the pair's scale, the quantised limbs); the
// warps multiply, keeping exact int32 sums per (tile, super-block), and fold them into fp32
// with the super-block's factors.  The warps of a row tile are summed in shared memory, T
// (the sum of x') is added, then the output scale and the store.

// Programmatic dependent launch: before griddepcontrol.wait a CTA only prefetches its
// sign rows into L2 (every input may be an output of the previous grid); the next grid
// is released after the wait.
#include <algorithm>

#include "ob_device.cuh"
#include "ob_internal.h"

#include "i8_block.cuh"

namespace ob {
namespace {

using namespace i8;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRT = 2;                       // row tiles per CTA
constexpr int kStride = kWarps / kRT;        // super-blocks between a warp's items
constexpr int kItems = 6;                    // items (super-blocks) a warp holds words for
constexpr int kMaxPairs = 3;                 // staging pairs per warp and chunk

template <int TOK>
constexpr int chunk_max() { return kMaxPairs * kWarps / TOK; }  // 24 (one token) or 12 super-blocks

template <int TOK, bool kVec>
__global__ void __launch_bounds__(kThreads) sign_gemm_i8_kernel(SignGemmArgs g, int64_t m0, int ch) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float tsum[TOK];
  __shared__ float red[kWarps][4][32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t n0 = (int64_t)blockIdx.x * (16 * kRT);
  const int64_t K = g.K, Wd = K / 32;
  const int64_t nsb = (K + kSbK - 1) / kSbK;
  const int64_t mt = min64(TOK, g.M - m0);

  if (g.l2_prefetch && warp == 0 && n0 < g.R) {
    const int64_t rows = min64(16 * kRT, g.R - n0);
    prefetch_block_l2(g.S + n0 * Wd, (uint64_t)(rows * Wd) * 4u, lane);
  }
  pdl_wait();
  pdl_launch_dependents();

  const Stage<TOK> st = Stage<TOK>::carve(dsm, ch);
  if (tid < TOK) tsum[tid] = 0.f;
  const int rt = warp % kRT;
  const int64_t row_g = n0 + 16 * rt + gq, row_h = row_g + 8;
  float tot[4] = {0.f, 0.f, 0.f, 0.f};

  for (int64_t sb0 = 0; sb0 < nsb; sb0 += ch) {
    const int chn = (int)min64(ch, nsb - sb0);
    // This warp's items of the chunk: super-blocks s = warp / 2 + 4 i.
    uint4 wg[kItems], wh[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int s = warp / kRT + it * kStride;
      wg[it] = make_uint4(0u, 0u, 0u, 0u);
      wh[it] = wg[it];
      if (s < chn) {
        const int64_t w0 = (sb0 + s) * kSbWords + 4 * tq;
        wg[it] = load_words<kVec>(g.S, g.R, Wd, row_g, w0);
        wh[it] = load_words<kVec>(g.S, g.R, Wd, row_h, w0);
      }
    }
    __syncthreads();  // the previous chunk's stage is no longer read
    // Staging: the pairs (token, super-block) p = warp, warp + 8, warp + 16, each with its own
    // scale.
    StageRaw raw[kMaxPairs];
#pragma unroll
    for (int k = 0; k < kMaxPairs; ++k) {
      const int p = warp + k * kWarps;
      if (p < TOK * chn) raw[k] = stage_load<false>(g, m0 + p % TOK, p % TOK < mt, (sb0 + p / TOK) * kSbK, lane);
    }
#pragma unroll
    for (int k = 0; k < kMaxPairs; ++k) {
      const int p = warp + k * kWarps;
      if (p < TOK * chn) stage_pair<TOK>(raw[k], p % TOK, st, p / TOK, lane);
    }
    __syncthreads();
    if (warp == kWarps - 1) {
#pragma unroll
      for (int m = 0; m < TOK; ++m) {
        const float t = chunk_sum<TOK>(st, chn, m, lane);
        if (lane == 0) tsum[m] += t;
      }
    }
    // Multiply: exact int32 sums per (tile, super-block), folded with the super-block's
    // factors.
    const int c0 = 2 * tq;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int s = warp / kRT + it * kStride;
      if (s < chn) {
        int acc[kChains][4];
#pragma unroll
        for (int j = 0; j < kChains; ++j)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[j][r] = 0;
        tile_sb(st.frag_at(s), wg[it], wh[it], acc, lane);
        const float* f = st.fold_at(s);
        const float f0 = f[c0], f1 = f[c0 + 1];
#pragma unroll
        for (int r = 0; r < 4; ++r) tot[r] = fmaf((float)combine(acc, r), (r & 1) ? f1 : f0, tot[r]);
      }
    }
    // Items past kItems (a chunk longer than kItems * 4 super-blocks) are not possible:
    // chunk_max() <= 24 = kItems * kStride.
  }

  // Sum the warps of each row tile, add T, scale, store.
#pragma unroll
  for (int r = 0; r < 4; ++r) red[warp][r][lane] = tot[r];
  __syncthreads();
  for (int idx = tid; idx < 16 * kRT * TOK; idx += kThreads) {
    const int r = idx % (16 * kRT), m = idx / (16 * kRT);
    const int64_t n = n0 + r;
    if (m >= mt || n >= g.R) continue;
    const int rtile = r >> 4, r16 = r & 15;
    const int gg = r16 & 7, hh = r16 >> 3;
    float v = tsum[m];
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) {
      const int col = kLimbs * m + l;
      const int src = 4 * gg + (col >> 1), reg = 2 * hh + (col & 1);
      for (int w = rtile; w < kWarps; w += kRT) v += red[w][reg][src];
    }
    v *= __ldg(g.oscale + n);
    const int64_t off = (m0 + m) * g.ldy + n;
    if (g.y_dtype == OB_OUT_F32)
      static_cast<float*>(g.Y)[off] = v;
    else
      static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(v);
  }
}

template <int TOK, bool kVec>
cudaError_t launch_tok(const SignGemmArgs& g, int64_t m0, const LaunchCtx& c) {
  const int64_t nsb = (g.K + kSbK - 1) / kSbK;
  const int ch = (int)std::min<int64_t>(nsb, chunk_max<TOK>());
  const size_t smem = Stage<TOK>::bytes(ch);
  auto kern = sign_gemm_i8_kernel<TOK, kVec>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((g.R + 16 * kRT - 1) / (16 * kRT)), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, g, m0, ch);
}

}  // namespace

cudaError_t launch_sign_gemm_i8(const SignGemmArgs& g, const LaunchCtx& c) {
  if (g.M == 0 || g.R == 0 || g.K == 0) return cudaSuccess;
  const bool vec = ((g.K / 32) % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.S) & 15) == 0);
  for (int64_t m0 = 0; m0 < g.M; m0 += kMaxTok) {
    const int64_t mt = std::min<int64_t>(kMaxTok, g.M - m0);
    cudaError_t e = mt == 1 ? (vec ? launch_tok<1, true>(g, m0, c) : launch_tok<1, false>(g, m0, c))
                            : (vec ? launch_tok<2, true>(g, m0, c) : launch_tok<2, false>(g, m0, c));
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace ob
