// mma_decode_block.cuh -- one 32-row block of a small-M sign product with warp-level MMA.
//
//   Y[m, n] = oscale[n] * sum_k (x[m, k] * iscale[k]) * s[n, k],   m0 <= m < m0 + TOK, n0 <= n < n0 + 32
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T.
// The mapping onto mma.sync.m16n8k16 is described in linear_mma_decode.cu.  Used by
// the per-call decode kernel (one CTA per block) and by the layer-stack kernel
// (persistent CTAs walking a list of blocks).
#pragma once

#include <cuda_bf16.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace mmad {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kRowTiles = 2;                 // m16 tiles per CTA
constexpr int kRowsPerCta = 16 * kRowTiles;  // 32
constexpr int kChunkWords = 16;              // 512 k per chunk

// Two A elements (k = c and c+16 of a packed word): bf16x2(b_c, b_c+16) with its
// two sign bits flipped where the packed bits are set.
__device__ __forceinline__ uint32_t unpack_pair(uint32_t w, int c, uint32_t bpair) {
  return ((w << (15 - c)) & 0x80008000u) ^ bpair;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Word w of row `row` of a warp's 32 x 16 word tile, at a 16-byte-group swizzle
// that makes the 8 rows one fragment reads fall in 8 different banks.
__host__ __device__ __forceinline__ int word_slot(int row, int w) {
  return row * kChunkWords + (w ^ (4 * ((row >> 1) & 3)));
}

// 16 bytes of activations.  Within one grid launch X is read-only for the per-call
// kernel (the read-only path is fine); the layer-stack kernel reads outputs that
// other CTAs of the same grid wrote before a grid barrier, so it reads through L2.
template <bool kCoherentX>
__device__ __forceinline__ uint4 load_x16(const uint16_t* p) {
  if constexpr (kCoherentX)
    return __ldcg(reinterpret_cast<const uint4*>(p));
  else
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// Dynamic shared memory of a block: per warp the B fragments of one chunk, then two
// word tiles (double buffer).
template <int TOK>
constexpr size_t dyn_smem_bytes() {
  return sizeof(uint2) * kWarps * kChunkWords * 2 * (TOK > 8 ? 2 : 1) * 32 +
         sizeof(uint32_t) * kWarps * 2 * kRowsPerCta * kChunkWords;
}

// Static shared memory of a block (declared __shared__ by the kernel).
template <int TOK>
struct BlockShared {
  float red[kWarps][kRowTiles][TOK > 8 ? 2 : 1][4][32];
  alignas(16) uint32_t bt[kWarps][kChunkWords][2][8];  // input-scale pairs per (word, step, t)
};

// The calling warp's word tiles (two buffers of 32 rows x 16 words) in the block's
// dynamic shared memory.
template <int TOK>
__device__ __forceinline__ uint32_t* warp_words(uint8_t* dsm, int warp) {
  constexpr int NN = TOK > 8 ? 2 : 1;
  uint32_t* swbase = reinterpret_cast<uint32_t*>(dsm + sizeof(uint2) * kWarps * kChunkWords * 2 * NN * 32);
  return swbase + warp * 2 * kRowsPerCta * kChunkWords;
}

// Request the calling warp's sign words of a chunk (32 rows x 16 words) into buffer `buf`
// of its word tiles `sw` (one cp.async group).
__device__ __forceinline__ void fetch_words(const SignGemmArgs& g, int64_t n0, bool vec, uint32_t* sw, int64_t chunk,
                                            int buf, int lane) {
  const int64_t Wd = g.K / 32;
  const int64_t nchunks = (Wd + kChunkWords - 1) / kChunkWords;
  uint32_t* dst = sw + buf * kRowsPerCta * kChunkWords;
  const int64_t w0 = chunk * kChunkWords;
  if (vec) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // 32 rows x 4 groups of 4 words = 128 copies per warp
      const int item = lane + 32 * i;
      const int row = item >> 2, q = item & 3;
      const int64_t n = n0 + row;
      const bool ok = n < g.R && chunk < nchunks && w0 + 4 * q < Wd;
      const uint32_t* src = g.S + (ok ? n * Wd + w0 + 4 * q : 0);
      cp_async16(dst + word_slot(row, 4 * q), src, ok);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) {  // 32 rows x 16 single words
      const int item = lane + 32 * i;
      const int row = item >> 4, w = item & 15;
      const int64_t n = n0 + row;
      const bool ok = n < g.R && chunk < nchunks && w0 + w < Wd;
      const uint32_t* src = g.S + (ok ? n * Wd + w0 + w : 0);
      cp_async4(dst + word_slot(row, w), src, ok);
    }
  }
  cp_async_commit();
}

// Y rows n0 .. n0+31 for tokens m0 .. m0+min(TOK, M-m0)-1.  All 256 threads call
// it; it ends with __syncthreads().  vec: the sign rows allow 16-byte copies.
// first_fetched: the caller has already issued fetch_words for each warp's first chunk
// (chunk = warp, buffer 0), e.g. before a programmatic-launch wait.
template <int TOK, bool kCoherentX>
__device__ __forceinline__ void block(const SignGemmArgs& g, int64_t m0, int64_t n0, bool vec, uint8_t* dsm,
                                      BlockShared<TOK>& shb, bool first_fetched = false) {
  constexpr int NN = TOK > 8 ? 2 : 1;
  constexpr int TOKN = TOK > 8 ? 8 : TOK;  // real tokens staged per n8 tile
  auto fb = reinterpret_cast<uint2 (*)[kChunkWords][2][NN][32]>(dsm);
  auto& red = shb.red;
  auto& bt = shb.bt;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;  // mma group / thread-in-group
  const int64_t K = g.K, Wd = K / 32;
  const int64_t mt = min64(TOK, g.M - m0);
  const int64_t nchunks = (Wd + kChunkWords - 1) / kChunkWords;
  uint32_t* sw = warp_words<TOK>(dsm, warp);
  auto fetch = [&](int64_t chunk, int buf) { fetch_words(g, n0, vec, sw, chunk, buf, lane); };

  // Stage one chunk for this warp: the B fragments (the activations, copied into
  // fragment order, no arithmetic) and the input-scale pairs that the A
  // fragments fold in.  Unit (word w, step s, tile nn) -> 32 lanes x 2 registers;
  // lane u of the warp builds unit u (+32).
  auto stage_x = [&](int64_t chunk) {
    constexpr int kUnits = kChunkWords * 2 * NN;
    {  // scale pairs: lane -> (w = lane/2, s = lane%2), 8 pairs (t = 0..3, c and c+4)
      const int w = lane >> 1, s = lane & 1;
      const int64_t kb = (chunk * kChunkWords + w) * 32 + 8 * s;
      uint4 o0 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u), o1 = o0;
      if (g.iscale && kb < K) {
        const float4* p4 = reinterpret_cast<const float4*>(g.iscale + kb);
        const float4 a0 = __ldg(p4), a1 = __ldg(p4 + 1), b0 = __ldg(p4 + 4), b1 = __ldg(p4 + 5);
        // bt[w][s][t] = {pair(c = 8s+t), pair(c + 4)}, pair(c) = (b[c], b[c+16])
        o0 = make_uint4(pack_bf16x2(a0.x, b0.x), pack_bf16x2(a1.x, b1.x), pack_bf16x2(a0.y, b0.y),
                        pack_bf16x2(a1.y, b1.y));
        o1 = make_uint4(pack_bf16x2(a0.z, b0.z), pack_bf16x2(a1.z, b1.z), pack_bf16x2(a0.w, b0.w),
                        pack_bf16x2(a1.w, b1.w));
      }
      uint4* dst = reinterpret_cast<uint4*>(&bt[warp][w][s][0]);
      dst[0] = o0;
      dst[1] = o1;
    }
#pragma unroll
    for (int u0 = 0; u0 < kUnits; u0 += 32) {
      const int u = u0 + lane;
      const int w = u / (2 * NN), s = (u / NN) & 1, nn = u % NN;
      const int64_t kb = (chunk * kChunkWords + w) * 32 + 8 * s;  // columns c = 8s .. 8s+7 of word w
      const bool kok = kb < K;
      uint4 xlo[TOKN], xhi[TOKN];
#pragma unroll
      for (int gg = 0; gg < TOKN; ++gg) {
        const int m = 8 * nn + gg;
        xlo[gg] = make_uint4(0, 0, 0, 0);
        xhi[gg] = make_uint4(0, 0, 0, 0);
        if (m < mt && kok) {
          const uint16_t* xr = g.X + (m0 + m) * K + kb;
          xlo[gg] = load_x16<kCoherentX>(xr);
          xhi[gg] = load_x16<kCoherentX>(xr + 16);
        }
      }
      // Lane (gg, t) of the fragment: b0 = (x[c], x[c+16]) with c = 8s+t, b1 = (x[c+4], x[c+20]),
      // token 8nn+gg: one byte permutation per register.
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) {
        uint4 out0 = make_uint4(0, 0, 0, 0), out1 = make_uint4(0, 0, 0, 0);
        if (gg < TOKN) {
          const uint4 lo = xlo[gg], hi = xhi[gg];
          out0.x = __byte_perm(lo.x, hi.x, 0x5410); out0.y = __byte_perm(lo.z, hi.z, 0x5410);
          out0.z = __byte_perm(lo.x, hi.x, 0x7632); out0.w = __byte_perm(lo.z, hi.z, 0x7632);
          out1.x = __byte_perm(lo.y, hi.y, 0x5410); out1.y = __byte_perm(lo.w, hi.w, 0x5410);
          out1.z = __byte_perm(lo.y, hi.y, 0x7632); out1.w = __byte_perm(lo.w, hi.w, 0x7632);
        }
        // Fragment slots of a unit are XOR-swizzled by the unit index so that the
        // 32 lanes (32 different units) do not all store to the same banks.
        uint4* dst = reinterpret_cast<uint4*>(&fb[warp][w][s][nn][4 * (gg ^ (u & 7))]);
        dst[0] = out0;
        dst[1] = out1;
      }
    }
  };

  constexpr int kSets = NN == 1 ? 4 : 2;  // independent accumulator chains
  float acc[kSets][kRowTiles][NN][4];
#pragma unroll
  for (int q = 0; q < kSets; ++q)
#pragma unroll
    for (int rt = 0; rt < kRowTiles; ++rt)
#pragma unroll
      for (int nn = 0; nn < NN; ++nn)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[q][rt][nn][i] = 0.f;

  int64_t chunk = warp;
  if (!first_fetched) fetch(chunk, 0);
  const int my_row = tid & (kRowsPerCta - 1);  // the output row this thread stores
  const float osc = (n0 + my_row < g.R) ? __ldg(g.oscale + n0 + my_row) : 0.f;
  int buf = 0;
  for (; chunk < nchunks; chunk += kWarps, buf ^= 1) {
    stage_x(chunk);
    if (chunk + kWarps < nchunks) {
      fetch(chunk + kWarps, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");  // this chunk's words have landed
    } else {
      cp_async_wait_all();
    }
    __syncwarp();
    const uint32_t* wt = sw + buf * kRowsPerCta * kChunkWords;
#pragma unroll
    for (int w = 0; w < kChunkWords; ++w) {
      uint32_t wr[kRowTiles][2];
#pragma unroll
      for (int rt = 0; rt < kRowTiles; ++rt)
#pragma unroll
        for (int h = 0; h < 2; ++h) wr[rt][h] = wt[word_slot(16 * rt + gq + 8 * h, w)];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int c0 = 8 * s + tq;
        const uint2 bp = *reinterpret_cast<const uint2*>(&bt[warp][w][s][2 * tq]);
        uint32_t a[kRowTiles][4];
#pragma unroll
        for (int rt = 0; rt < kRowTiles; ++rt) {
          a[rt][0] = unpack_pair(wr[rt][0], c0, bp.x);
          a[rt][1] = unpack_pair(wr[rt][1], c0, bp.x);
          a[rt][2] = unpack_pair(wr[rt][0], c0 + 4, bp.y);
          a[rt][3] = unpack_pair(wr[rt][1], c0 + 4, bp.y);
        }
#pragma unroll
        for (int nn = 0; nn < NN; ++nn) {
          const int unit = (w * 2 + s) * NN + nn;
          const uint2 b = fb[warp][w][s][nn][lane ^ (4 * (unit & 7))];
#pragma unroll
          for (int rt = 0; rt < kRowTiles; ++rt) mma_16816(acc[w % kSets][rt][nn], a[rt], b.x, b.y);
        }
      }
    }
    __syncwarp();  // fb and this word buffer are rewritten two chunks on
  }
  cp_async_wait_all();

  // Sum the warps' partial tiles, scale, store.
#pragma unroll
  for (int rt = 0; rt < kRowTiles; ++rt)
#pragma unroll
    for (int nn = 0; nn < NN; ++nn)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v = acc[0][rt][nn][i];
#pragma unroll
        for (int q = 1; q < kSets; ++q) v += acc[q][rt][nn][i];
        red[warp][rt][nn][i][lane] = v;
      }
  __syncthreads();
  const int outputs = kRowsPerCta * 8 * NN;
  for (int idx = tid; idx < outputs; idx += kThreads) {
    const int r = idx % kRowsPerCta;   // == my_row: weight row within the CTA (fastest: coalesced stores)
    const int m = idx / kRowsPerCta;   // token
    const int64_t n = n0 + r;
    if (m >= mt || n >= g.R) continue;
    const int rt = r >> 4, rho = r & 15;
    const int gg = rho & 7, hh = rho >> 3;
    const int nn = m >> 3, col = m & 7;
    const int lane_src = 4 * gg + (col >> 1);
    const int reg = 2 * hh + (col & 1);
    float v = 0.f;
#pragma unroll
    for (int wp = 0; wp < kWarps; ++wp) v += red[wp][rt][nn][reg][lane_src];
    v *= osc;
    const int64_t off = (m0 + m) * g.ldy + n;
    if (g.y_dtype == OB_OUT_F32)
      static_cast<float*>(g.Y)[off] = v;
    else
      static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(v);
  }
  __syncthreads();  // the next block on this CTA reuses the shared buffers
}

}  // namespace mmad
}  // namespace ob
