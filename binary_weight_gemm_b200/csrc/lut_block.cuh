// lut_block.cuh -- one 32-row block of a one-token sign product by table lookup.
//
//   y[n] = oscale[n] * sum_k (x[k] * iscale[k]) * s[n, k],   row_base <= n < row_base + 32
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": y = [(x ⊙ b^T) W_sign^T] ⊙ a^T.
// For every group of 4 consecutive k the CTA tabulates the 16 signed sums
// +-x'_0 +-x'_1 +-x'_2 +-x'_3 (x' = x ⊙ b) in shared memory, so each packed nibble
// costs one shared-memory load and one add instead of four select/adds.  Table
// layout: entry v of group (lane group c, word q, nibble j) sits at
// v * 32*Q*8 + (8q + j) * 32 + c, so lane c always reads bank c.  8 warps x 4 rows.
// Used by the per-call one-token kernel (one CTA per block).
#pragma once

#include <cuda_bf16.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace lutb {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerBlock = kWarps * kRowsPerWarp;  // 32

// Q packed words per lane per chunk: 4 when rows allow 16-byte loads, else 1.
template <int Q>
constexpr size_t smem_bytes() {
  return sizeof(float) * 16 * 32 * Q * 8;
}

// 8 bytes of activations: through the read-only path in the per-call kernel, through
// L2 in the layer-stack kernel (other CTAs of that grid wrote them).
template <bool kCoherentX>
__device__ __forceinline__ uint2 load_x8(const uint16_t* p) {
  if constexpr (kCoherentX)
    return __ldcg(reinterpret_cast<const uint2*>(p));
  else
    return __ldg(reinterpret_cast<const uint2*>(p));
}

// This lane's sign words of chunk c0 (32 lanes x Q words) for the warp's rows starting at row0.
template <int Q>
__device__ __forceinline__ void load_signs(const SignGemmArgs& g, int64_t row0, int64_t c0,
                                           uint32_t (&wq)[kRowsPerWarp][Q], int lane) {
  const int64_t Wd = g.K / 32, G = (Wd + Q - 1) / Q;
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
}

// The output scales of the warp's rows.
__device__ __forceinline__ void load_oscale(const SignGemmArgs& g, int64_t row0, float (&osc)[kRowsPerWarp]) {
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) osc[r] = (row0 + r < g.R) ? __ldg(g.oscale + row0 + r) : 0.f;
}

// First row of the calling warp's rows in a block.
__device__ __forceinline__ int64_t warp_row0(int64_t row_base) { return row_base + (threadIdx.x >> 5) * kRowsPerWarp; }

// Y[m0, row_base .. row_base + 31]; all 256 threads call it; it ends with __syncthreads().
// wq0: the lane's sign words of the first chunk and osc: the output scales, both loaded by
// the caller with load_signs / load_oscale (before or after the programmatic-launch wait).
template <int Q, bool kCoherentX>
__device__ __forceinline__ void block(const SignGemmArgs& g, int64_t m0, int64_t row_base, float* lut,
                                      const uint32_t (&wq0)[kRowsPerWarp][Q], const float (&osc)[kRowsPerWarp]) {
  constexpr int kGroups = 32 * Q * 8;  // nibble groups per chunk (4 k each)
  const int lane = threadIdx.x & 31;
  const int64_t K = g.K, Wd = K / 32, G = (Wd + Q - 1) / Q;
  const int64_t row0 = warp_row0(row_base);
  float acc[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) acc[r] = 0.f;

  for (int64_t c0 = 0; c0 < G; c0 += 32) {
    // 1. This lane's sign words for every row of the warp.
    uint32_t wq[kRowsPerWarp][Q];
    if (c0 == 0) {
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int q = 0; q < Q; ++q) wq[r][q] = wq0[r][q];
    } else {
      load_signs<Q>(g, row0, c0, wq, lane);
    }
    // 2. Tabulate this chunk: thread t builds groups with c = t % 32, (8q+j) = t/32 + 8i.
    constexpr int kPerThread = kGroups / kThreads;  // 4 (Q = 4) or 1 (Q = 1)
    float x[kPerThread][4];
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const int c = threadIdx.x & 31, qj = (threadIdx.x >> 5) + 8 * i;
      const int q = qj >> 3, j = qj & 7;
      const int64_t k = (c0 + c) * Q * 32 + q * 32 + 4 * j;
      float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
      uint2 xv = make_uint2(0u, 0u);
      if (k < K && (c0 + c) < G) {
        sc = g.iscale ? __ldg(reinterpret_cast<const float4*>(g.iscale + k)) : make_float4(1.f, 1.f, 1.f, 1.f);
        xv = load_x8<kCoherentX>(g.X + m0 * K + k);
      }
      x[i][0] = __uint_as_float(xv.x << 16) * sc.x;
      x[i][1] = __uint_as_float(xv.x & 0xFFFF0000u) * sc.y;
      x[i][2] = __uint_as_float(xv.y << 16) * sc.z;
      x[i][3] = __uint_as_float(xv.y & 0xFFFF0000u) * sc.w;
    }
    __syncthreads();  // the previous chunk's readers are done with the table
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const int c = threadIdx.x & 31, qj = (threadIdx.x >> 5) + 8 * i;
      const int slot = qj * 32 + c;
      // bit b of v set <=> sign of x_b is -1
      const float p[4] = {x[i][0] + x[i][1], -x[i][0] + x[i][1], x[i][0] - x[i][1], -x[i][0] - x[i][1]};
      const float h[4] = {x[i][2] + x[i][3], -x[i][2] + x[i][3], x[i][2] - x[i][3], -x[i][2] - x[i][3]};
#pragma unroll
      for (int v = 0; v < 16; ++v) lut[v * kGroups + slot] = p[v & 3] + h[v >> 2];
    }
    __syncthreads();
    // 3. One table load and one add per packed nibble.
    const uint32_t lane_off = (uint32_t)lane * 4u;  // byte offset of bank `lane`
    const char* lbase = reinterpret_cast<const char*>(lut);
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
#pragma unroll
      for (int q = 0; q < Q; ++q) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // byte offset of entry v: v * kGroups * 4 = v << log2(kGroups * 4)
          constexpr int kShift = (Q == 4) ? 12 : 10;  // log2(kGroups * 4)
          const uint32_t w = wq[r][q];
          const int sh = kShift - 4 * j;
          const uint32_t vb = sh >= 0 ? (w << sh) : (w >> (-sh));
          const uint32_t off = (vb & (0xFu << kShift)) | lane_off;
          acc[r] += *reinterpret_cast<const float*>(lbase + off + (q * 8 + j) * 32 * 4);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    float v = acc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int64_t n = row0 + r;
    if (lane == 0 && n < g.R) {
      v *= osc[r];
      const int64_t off = m0 * g.ldy + n;
      if (g.y_dtype == OB_OUT_F32)
        static_cast<float*>(g.Y)[off] = v;
      else
        static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(v);
    }
  }
  __syncthreads();  // the next block on this CTA rebuilds the table
}

}  // namespace lutb
}  // namespace ob
