// linear_stack_f8.cu -- a list of one- or two-token sign-product layers in one persistent
// launch, on fp8 tensor cores (f8_block.cuh).
//
// Each layer is  Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T  ("1bit量化", blog.zerodtree.com,
// "proposition 1"); a decoder applies such layers one after another.  The list is
// walked by one cooperative grid (one CTA per SM), as in linear_stack.cu, with the
// layers between two grid barriers (a barrier group) run back to back.
//
//  * Work split.  A group's rows, in 16-row tiles, are cut into one contiguous range
//    per CTA, so a CTA sees at most a few layers per group and stages the activation
//    fragments (x ⊙ b in e4m3 limbs) of each such layer once, for all its tiles.
//  * Within a layer, the CTA's eight warps take the super-blocks (512 k) of every tile
//    of its range round robin (super-block s goes to warp s mod 8), fold each into
//    fp32 per tile, and leave the per-warp tile sums in shared memory; the epilogue
//    adds them in warp order (deterministic), adds the sum of x', applies a and stores.
//  * Weights do not depend on activations: before computing a group, each CTA
//    prefetches into L2 the sign rows of its range of the next group and the scale
//    vectors, so they stream in while this group computes and the grid waits at the
//    barrier.  Packed words are then loaded into registers four items ahead.
//  * The barrier is the bounded grid barrier of stack_common.cuh.
#include <algorithm>
#include <cstring>

#include "f8_block.cuh"
#include "stack_common.cuh"

namespace ob {
namespace {

using namespace f8;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTiles = 12;                  // tiles of one layer a CTA reduces at once
constexpr int kItems = 4;                      // items whose words a warp holds
constexpr size_t kStageBudget = 96 * 1024;     // staged fragments (24 super-blocks at TOK <= 2)

template <int TOK>
constexpr size_t red_bytes() {
  return sizeof(float) * kMaxTiles * kWarps * Stage<TOK>::NT * 4 * 32;
}

template <int TOK>
int chunk_sbs_max() {
  return (int)(kStageBudget / Stage<TOK>::bytes_per_sb());
}

__device__ __forceinline__ int64_t tiles_of(const StackLayer& L) { return (L.N + 15) / 16; }

// The contiguous range of group tiles [lo, hi) CTA c of G owns, out of T.
__device__ __forceinline__ void tile_range(int64_t T, int c, int G, int64_t* lo, int64_t* hi) {
  *lo = T * c / G;
  *hi = T * (c + 1) / G;
}

// L2 prefetch of what this CTA reads of the group [l, e): its sign rows and the scale
// vectors of the layers its range touches.  One warp.
__device__ void prefetch_group_f8(const StackParams& p, int l, int e, int lane) {
  int64_t T = 0;
  for (int li = l; li < e; ++li) T += tiles_of(p.L[li]);
  int64_t lo, hi;
  tile_range(T, blockIdx.x, gridDim.x, &lo, &hi);
  int64_t base = 0;
  for (int li = l; li < e && base < hi; ++li) {
    const StackLayer& L = p.L[li];
    const int64_t nt = tiles_of(L);
    const int64_t a = max(lo, base), b = min(hi, base + nt);
    if (a < b) {
      const int64_t Wd = L.K / 32, r0 = (a - base) * 16, r1 = min64((b - base) * 16, L.N);
      if (L.vec) prefetch_block_l2(L.S + r0 * Wd, (uint64_t)((r1 - r0) * Wd) * 4u, lane);
      if (L.iscale) prefetch_block_l2(L.iscale, (uint64_t)L.K * 4u, lane);
      prefetch_block_l2(L.oscale + r0, (uint64_t)(r1 - r0) * 4u, lane);
    }
    base += nt;
  }
}

// Tiles [t0, t0 + nt) (nt <= kMaxTiles) of layer L: stage, multiply, reduce, store.
template <int TOK, bool kVec>
__device__ void layer_tiles(const StackParams& p, const StackLayer& L, int64_t t0, int nt, int ch, uint8_t* dsm,
                            float* tsum) {
  constexpr int NT = Stage<TOK>::NT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  SignGemmArgs g{L.X, p.M, L.K, L.S, L.N, L.iscale, L.oscale, L.Y, L.N, L.y_dtype, 0};
  const int64_t K = L.K, Wd = K / 32, nsb = (K + kSbK - 1) / kSbK;
  const int64_t mt = min64(TOK, p.M);
  const Stage<TOK> st = Stage<TOK>::carve(dsm, ch);
  float* red = reinterpret_cast<float*>(dsm + Stage<TOK>::bytes_per_sb() * (size_t)ch);
  __syncthreads();  // the previous layer's epilogue no longer reads red / tsum
  if (tid < TOK) tsum[tid] = 0.f;

  for (int64_t sb0 = 0; sb0 < nsb; sb0 += ch) {
    const int chn = (int)min64(ch, nsb - sb0);
    // This warp's items of the chunk: (tile i, super-block s) for s = warp, warp + 8, ...
    // in the order (i, s); item index q -> tile q / per, slot warp + 8 (q % per).
    const int per = chn > warp ? (chn - warp + kWarps - 1) / kWarps : 0;
    const int items = per * nt;
    uint4 wg[kItems], wh[kItems];
    auto load_batch = [&](int q0) {
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        wg[it] = make_uint4(0u, 0u, 0u, 0u);
        wh[it] = wg[it];
        const int q = q0 + it;
        if (q < items) {
          const int i = q / per, s = warp + kWarps * (q % per);
          const int64_t row = (t0 + i) * 16 + gq, w0 = (sb0 + s) * kSbWords + 4 * tq;
          wg[it] = load_words<kVec>(L.S, L.N, Wd, row, w0);
          wh[it] = load_words<kVec>(L.S, L.N, Wd, row + 8, w0);
        }
      }
    };
    load_batch(0);
    __syncthreads();  // the previous chunk's fragments are no longer read
    for (int pp = warp; pp < TOK * chn; pp += 2 * kWarps) {
      const int p2 = pp + kWarps;
      const StageRaw r0 = stage_load<true>(g, pp % TOK, pp % TOK < mt, (sb0 + pp / TOK) * kSbK, lane);
      StageRaw r1;
      if (p2 < TOK * chn) r1 = stage_load<true>(g, p2 % TOK, p2 % TOK < mt, (sb0 + p2 / TOK) * kSbK, lane);
      stage_convert<TOK>(r0, pp % TOK, st, pp / TOK, lane);
      if (p2 < TOK * chn) stage_convert<TOK>(r1, p2 % TOK, st, p2 / TOK, lane);
    }
    __syncthreads();
    float tot[NT][4];
    for (int q0 = 0; q0 < items; q0 += kItems) {
#pragma unroll
      for (int it = 0; it < kItems; ++it) {
        const int q = q0 + it;
        if (q < items) {
          const int i = q / per, k = q % per;
          if (k == 0) {
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
              for (int r = 0; r < 4; ++r) tot[a][r] = 0.f;
          }
          tile_sb<TOK>(st, warp + kWarps * k, wg[it], wh[it], tot, lane);
          if (k == per - 1) {  // the tile's last item of this chunk: into its slot
            float* dst = red + (size_t)(i * kWarps + warp) * NT * 128;
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                float* d = dst + (a * 4 + r) * 32 + lane;
                *d = sb0 == 0 ? tot[a][r] : *d + tot[a][r];
              }
          }
        }
      }
      if (q0 + kItems < items) load_batch(q0 + kItems);
    }
    // A warp with no item in this chunk (short K) leaves zeros in the first chunk.
    if (items == 0 && sb0 == 0) {
      for (int i = 0; i < nt; ++i) {
        float* dst = red + (size_t)(i * kWarps + warp) * NT * 128;
        for (int r = lane; r < NT * 128; r += 32) dst[r] = 0.f;
      }
    }
    if (tid < TOK) {
      float acc = tsum[tid];
      for (int sl = 0; sl < chn; ++sl) acc += st.tsb[sl * TOK + tid];
      tsum[tid] = acc;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < nt * 16 * TOK; idx += kThreads) {
    const int r = idx % (nt * 16), m = idx / (nt * 16);
    const int64_t n = t0 * 16 + r;
    if (m >= mt || n >= L.N) continue;
    const int i = r >> 4, r16 = r & 15;
    const int gg = r16 & 7, hh = r16 >> 3;
    float v = tsum[m];
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) {
      const int col = kLimbs * m + l;
      const int a = col >> 3, cn = col & 7;
      const int src = 4 * gg + (cn >> 1), reg = 2 * hh + (cn & 1);
      for (int w = 0; w < kWarps; ++w) v += red[(size_t)(i * kWarps + w) * NT * 128 + (a * 4 + reg) * 32 + src];
    }
    v *= __ldg(L.oscale + n);
    const int64_t off = (int64_t)m * L.N + n;
    if (L.y_dtype == OB_OUT_F32)
      static_cast<float*>(L.Y)[off] = v;
    else
      static_cast<__nv_bfloat16*>(L.Y)[off] = __float2bfloat16_rn(v);
  }
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 1) sign_stack_f8_kernel(const __grid_constant__ StackParams p, int ch) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float tsum[TOK];
  __shared__ int s_ok;
  const int G = gridDim.x, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int e = group_end(p, 0);
  if (warp == 0) prefetch_group_f8(p, 0, e, lane);
  pdl_wait();  // the first layers' inputs may come from the previous grid in the stream
  unsigned barriers = 0;
  for (int l = 0; l < p.n;) {
    const int e2 = e < p.n ? group_end(p, e) : e;
    if (warp == 0 && e < p.n) prefetch_group_f8(p, e, e2, lane);
    int64_t T = 0;
    for (int li = l; li < e; ++li) T += tiles_of(p.L[li]);
    int64_t lo, hi;
    tile_range(T, c, G, &lo, &hi);
    int64_t base = 0;
    for (int li = l; li < e && base < hi; ++li) {
      const StackLayer& L = p.L[li];
      const int64_t ntl = tiles_of(L);
      int64_t a = max(lo, base) - base;
      const int64_t b = min(hi, base + ntl) - base;
      for (; a < b; a += kMaxTiles) {
        const int nt = (int)min64(kMaxTiles, b - a);
        if (L.vec)
          layer_tiles<TOK, true>(p, L, a, nt, ch, dsm, tsum);
        else
          layer_tiles<TOK, false>(p, L, a, nt, ch, dsm, tsum);
      }
      base += ntl;
    }
    l = e;
    e = e2;
    if (l < p.n) {
      ++barriers;
      if (!grid_barrier(p.bar, barriers * (unsigned)G, p.err, &s_ok)) return;
    }
  }
}

template <int TOK>
cudaError_t launch_f8_tok(const StackParams& prm, const LaunchCtx& c) {
  auto kern = sign_stack_f8_kernel<TOK>;
  int64_t max_k = 32;
  for (int i = 0; i < prm.n; ++i) max_k = std::max<int64_t>(max_k, prm.L[i].K);
  const int ch = (int)std::min<int64_t>(chunk_sbs_max<TOK>(), (max_k + kSbK - 1) / kSbK);
  const size_t smem = Stage<TOK>::bytes_per_sb() * (size_t)ch + red_bytes<TOK>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)c.num_sms, 1, 1);  // one CTA per SM: all resident (cooperative)
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, prm, ch);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stack_f8(const StackParams& prm, const LaunchCtx& c) {
  return prm.M == 1 ? launch_f8_tok<1>(prm, c) : launch_f8_tok<2>(prm, c);
}

}  // namespace ob
