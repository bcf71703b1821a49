// linear_f8.cu -- small-M sign product on fp8 tensor cores (f8_block.cuh), one call.
//
//   Y[m, n] = oscale[n] * sum_k (x[m, k] * iscale[k]) * s[n, k],   M <= 16 per pass
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T;
// each of DBF's two sign products ("Addition is almost all you need ...",
// "Methodologie") is one call.
//
// A CTA owns RT row tiles (16 rows each) and all of K.  K is taken in chunks of
// super-blocks (512 k) that fit shared memory: the CTA's eight warps first stage the
// chunk's activation fragments (one warp per (token, super-block)), then each warp
// multiplies its row tile (warp % RT) by its super-blocks of the chunk
// (warp / RT, + 8 / RT, ...), loading the next item's packed words while it works on
// the current one.  Partial tiles of the warps of one row tile are summed in shared
// memory, T (the sum of x') is added, then the output scale and the store.
//
// Programmatic dependent launch: before griddepcontrol.wait a CTA only prefetches its
// sign rows into L2 (every input may be an output of the previous grid); the next
// grid is released after the wait.
#include <algorithm>

#include "ob_device.cuh"
#include "ob_internal.h"

#include "f8_block.cuh"

namespace ob {
namespace {

using namespace f8;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr size_t kStageBudget = 96 * 1024;  // shared memory for staged fragments
constexpr int kItems = 4;                    // (row tile, super-block) items whose words a warp holds

template <int TOK>
int chunk_sbs(int64_t nsb) {
  const int64_t fit = (int64_t)(kStageBudget / Stage<TOK>::bytes_per_sb());
  return (int)std::max<int64_t>(1, std::min<int64_t>(nsb, fit));
}

template <int TOK, int RT>
constexpr size_t red_bytes() {
  return sizeof(float) * kWarps * Stage<TOK>::NT * 4 * 32;
}

template <int TOK, int RT, bool kVec>
__global__ void __launch_bounds__(kThreads) sign_gemm_f8_kernel(SignGemmArgs g, int64_t m0, int ch) {
  constexpr int NT = Stage<TOK>::NT;
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float tsum[TOK];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int64_t n0 = (int64_t)blockIdx.x * (16 * RT);
  const int64_t K = g.K, Wd = K / 32;
  const int64_t nsb = (K + kSbK - 1) / kSbK;
  const int64_t mt = min64(TOK, g.M - m0);

  if (g.l2_prefetch && warp == 0 && n0 < g.R) {
    const int64_t rows = min64(16 * RT, g.R - n0);
    prefetch_block_l2(g.S + n0 * Wd, (uint64_t)(rows * Wd) * 4u, lane);
  }
  pdl_wait();
  pdl_launch_dependents();

  const Stage<TOK> st = Stage<TOK>::carve(dsm, ch);
  float* red = reinterpret_cast<float*>(dsm + Stage<TOK>::bytes_per_sb() * (size_t)ch);
  if (tid < TOK) tsum[tid] = 0.f;

  const int rt = warp % RT;
  constexpr int kStride = kWarps / RT;  // super-blocks between a warp's items
  const int64_t row_g = n0 + 16 * rt + gq, row_h = row_g + 8;
  float tot[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) tot[nt][r] = 0.f;

  for (int64_t sb0 = 0; sb0 < nsb; sb0 += ch) {
    const int chn = (int)min64(ch, nsb - sb0);
    int s = warp / RT;
    // The packed words of this warp's first kItems items of the chunk are requested
    // before the staging, so that they are in flight while it runs.
    uint4 wg[kItems], wh[kItems];
    auto load_batch = [&](int s_first) {
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int si = s_first + it * kStride;
        wg[it] = make_uint4(0u, 0u, 0u, 0u);
        wh[it] = wg[it];
        if (si < chn) {
          const int64_t w0 = (sb0 + si) * kSbWords + 4 * tq;
          wg[it] = load_words<kVec>(g.S, g.R, Wd, row_g, w0);
          wh[it] = load_words<kVec>(g.S, g.R, Wd, row_h, w0);
        }
      }
    };
    load_batch(s);
    __syncthreads();  // the previous chunk's fragments are no longer read
    // Staging: (token, super-block) pairs dealt to warps; each warp issues the loads of
    // two pairs before converting either.
    for (int p = warp; p < TOK * chn; p += 2 * kWarps) {
      const int p2 = p + kWarps;
      const StageRaw r0 = stage_load<false>(g, m0 + p % TOK, p % TOK < mt, (sb0 + p / TOK) * kSbK, lane);
      StageRaw r1;
      if (p2 < TOK * chn) r1 = stage_load<false>(g, m0 + p2 % TOK, p2 % TOK < mt, (sb0 + p2 / TOK) * kSbK, lane);
      stage_convert<TOK>(r0, p % TOK, st, p / TOK, lane);
      if (p2 < TOK * chn) stage_convert<TOK>(r1, p2 % TOK, st, p2 / TOK, lane);
    }
    __syncthreads();
    for (; s < chn; s += kItems * kStride) {
#pragma unroll
      for (int it = 0; it < kItems; ++it)
        if (s + it * kStride < chn) tile_sb<TOK>(st, s + it * kStride, wg[it], wh[it], tot, lane);
      if (s + kItems * kStride < chn) load_batch(s + kItems * kStride);
    }
    if (tid < TOK) {
      float acc = tsum[tid];
      for (int sl = 0; sl < chn; ++sl) acc += st.tsb[sl * TOK + tid];
      tsum[tid] = acc;
    }
  }

  // Sum the warps of each row tile, add T, scale, store.
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) red[((warp * NT + nt) * 4 + r) * 32 + lane] = tot[nt][r];
  __syncthreads();
  for (int idx = tid; idx < 16 * RT * TOK; idx += kThreads) {
    const int r = idx % (16 * RT), m = idx / (16 * RT);
    const int64_t n = n0 + r;
    if (m >= mt || n >= g.R) continue;
    const int rtile = r >> 4, r16 = r & 15;
    const int gg = r16 & 7, hh = r16 >> 3;
    float v = tsum[m];
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) {
      const int col = kLimbs * m + l;
      const int nt = col >> 3, cn = col & 7;
      const int src = 4 * gg + (cn >> 1), reg = 2 * hh + (cn & 1);
      for (int w = rtile; w < kWarps; w += RT) v += red[((w * NT + nt) * 4 + reg) * 32 + src];
    }
    v *= __ldg(g.oscale + n);
    const int64_t off = (m0 + m) * g.ldy + n;
    if (g.y_dtype == OB_OUT_F32)
      static_cast<float*>(g.Y)[off] = v;
    else
      static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(v);
  }
}

template <int TOK, int RT, bool kVec>
cudaError_t launch_tok(const SignGemmArgs& g, int64_t m0, const LaunchCtx& c) {
  const int64_t nsb = (g.K + kSbK - 1) / kSbK;
  const int ch = chunk_sbs<TOK>(nsb);
  const size_t smem = Stage<TOK>::bytes_per_sb() * (size_t)ch + red_bytes<TOK, RT>();
  auto kern = sign_gemm_f8_kernel<TOK, RT, kVec>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((g.R + 16 * RT - 1) / (16 * RT)), 1, 1);
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

template <bool kVec>
cudaError_t launch_vec(const SignGemmArgs& g, int64_t m0, int64_t mt, const LaunchCtx& c) {
  if (mt == 1) return launch_tok<1, 2, kVec>(g, m0, c);
  if (mt == 2) return launch_tok<2, 2, kVec>(g, m0, c);
  if (mt <= 4) return launch_tok<4, 4, kVec>(g, m0, c);
  if (mt <= 8) return launch_tok<8, 4, kVec>(g, m0, c);
  return launch_tok<16, 8, kVec>(g, m0, c);
}

}  // namespace

cudaError_t launch_sign_gemm_f8(const SignGemmArgs& g, const LaunchCtx& c) {
  if (g.M == 0 || g.R == 0 || g.K == 0) return cudaSuccess;
  const bool vec = ((g.K / 32) % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.S) & 15) == 0);
  for (int64_t m0 = 0; m0 < g.M; m0 += 16) {
    const int64_t mt = std::min<int64_t>(16, g.M - m0);
    cudaError_t e = vec ? launch_vec<true>(g, m0, mt, c) : launch_vec<false>(g, m0, mt, c);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace ob
