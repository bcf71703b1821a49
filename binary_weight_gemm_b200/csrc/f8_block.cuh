// f8_block.cuh -- the sign product on fp8 tensor cores: packed signs become e4m3
// operands with one AND per four weights.
//
//   Y[m, n] = oscale[n] * sum_k x'[m, k] s[n, k],   x' = x ⊙ iscale,  s = 1 - 2 bit
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T;
// "Addition is almost all you need ..." (gist.science), "Methodologie": a product
// with a +/-1 matrix needs no multiplications.  Here the multiplications are the
// tensor core's, and the cost of getting the signs there is what is minimised.
//
// Identity used: sum_k s_k x'_k = T - 2 sum_k bit_k x'_k, with T = sum_k x'_k.  The
// masked sum sum_k bit_k x'_k is a dot product of a 0/1 matrix with x', computed by
// mma.sync.m16n8k32 with e4m3 operands (fp32 accumulation; checked exact to fp32
// rounding on B200, subnormal operands included):
//
//  * A (16 rows x 32 k, weights): byte i of register R_j of a packed word w is bit
//    8i + j of w, left where it is: R_j = (j < 4 ? w : w >> 4) & (0x01010101 << (j & 3)).
//    An e4m3 byte with the single bit p (p < 4) set is the number 2^(p - 9), so
//    R_j holds bit_k * c_j with c_j = 2^((j & 3) - 9): one AND per four weights
//    (plus one shift per word).
//  * B (32 k x 8 columns, activations): x'_k / c_j, times a power-of-two scale
//    sigma chosen per token and per 512 k so that the values sit in e4m3 range,
//    split into three e4m3 limbs (hi, then the residual times 16, twice) placed in
//    three accumulator columns; about 12 significant bits.  A column n = 3 m + l
//    holds limb l of token m.
//  * The product A B is then sum_k bit_k x'_k sigma 16^l per column.  After every
//    512 k the accumulators are folded into fp32 totals with the factor
//    -2 / (sigma 16^l); T is added in the epilogue.  Columns past 3 M are never
//    staged and never read: an MMA's output column depends only on its own B column.
//
// Fragment correspondence (PTX ISA, mma.m16n8k32 .e4m3): lane (g, t) holds A rows g
// and g+8, k-slots 4t + i (a0, a1) and 16 + 4t + i (a2, a3), and B column g,
// k-slots 4t + i (b0) and 16 + 4t + i (b1).  A super-block is 512 k = 16 packed
// words per row; lane t of a quad owns words 4t .. 4t+3 (one 16-byte load per row).
// MMA (e, u) of a super-block (e, u = 0..3) takes a0 = R_2u, a2 = R_2u+1 of word
// 4t + e of row g (a1, a3: row g+8), so k-slot 4t + i is k = 32 (4t + e) + 8 i + 2u
// and k-slot 16 + 4t + i is the same k + 1.  The B fragments are staged in shared
// memory in exactly that order, [e][u][n-tile][lane] as uint2 (b0, b1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace f8 {

constexpr int kLimbs = 3;
constexpr int kSbK = 512;                 // k per super-block
constexpr int kSbWords = kSbK / 32;       // packed words per row per super-block
constexpr int kFragWords = 4 * 4 * 32 * 2;  // 32-bit words of B fragments per (super-block, n-tile)

__host__ __device__ constexpr int n_tiles(int tok) { return (kLimbs * tok + 7) / 8; }

__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Register R_j of a packed word w (w4 = w >> 4): bit 8i + j of w in byte i, at bit j & 3.
__device__ __forceinline__ uint32_t lanes_of(uint32_t w, uint32_t w4, int j) {
  return (j < 4 ? w : w4) & (0x01010101u << (j & 3));
}

// Two fp32 to two e4m3 (round to nearest even, saturating): x.x in the low byte.
__device__ __forceinline__ uint32_t to_e4m3x2(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float2 from_e4m3x2(uint32_t v) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// Shared-memory layout of a staged chunk of `ch` super-blocks for TOK tokens.
template <int TOK>
struct Stage {
  static constexpr int NT = n_tiles(TOK);
  uint32_t* frag;  // [ch][e][u][NT][lane][2]
  float* fcol;     // [ch][NT * 8]: fold factor of each accumulator column
  float* tsb;      // [ch][TOK]: sum of x' over the super-block, per token
  __device__ __forceinline__ uint32_t* frag_at(int s) const { return frag + (size_t)s * NT * kFragWords; }
  static __host__ __device__ constexpr size_t bytes_per_sb() {
    return sizeof(uint32_t) * NT * kFragWords + sizeof(float) * NT * 8 + sizeof(float) * TOK;
  }
  __device__ static Stage carve(uint8_t* base, int ch) {
    Stage st;
    st.frag = reinterpret_cast<uint32_t*>(base);
    st.fcol = reinterpret_cast<float*>(base + sizeof(uint32_t) * (size_t)ch * NT * kFragWords);
    st.tsb = st.fcol + (size_t)ch * NT * 8;
    return st;
  }
};

// The raw inputs one lane needs to stage a (token, super-block): x (bf16) and the input
// scale at k = kbase + 32 q + 8 i + j, q = lane / 2, j = 4 (lane & 1) .. + 3, i = 0..3.
struct StageRaw {
  uint2 x[4];
  float4 sc[4];
};

// Issue the loads of one (token, super-block) (zeros when !live or past K).
template <bool kCoherentX>
__device__ __forceinline__ StageRaw stage_load(const SignGemmArgs& g, int64_t m_glob, bool live, int64_t kbase,
                                               int lane) {
  const int q = lane >> 1, jh = (lane & 1) * 4;
  const int64_t K = g.K;
  StageRaw r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k0 = kbase + 32 * q + 8 * i + jh;
    r.sc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    r.x[i] = make_uint2(0u, 0u);
    if (live && k0 < K) {  // K % 32 == 0: the four k are all in range or all out
      r.sc[i] = g.iscale ? __ldg(reinterpret_cast<const float4*>(g.iscale + k0)) : make_float4(1.f, 1.f, 1.f, 1.f);
      const uint2* px = reinterpret_cast<const uint2*>(g.X + m_glob * K + k0);
      r.x[i] = kCoherentX ? __ldcg(px) : __ldg(px);
    }
  }
  return r;
}

// One warp turns the loaded inputs of token m into slot s of the stage: the three e4m3
// limbs of every B register, the columns' fold factors and the super-block's sum of x'.
template <int TOK>
__device__ __forceinline__ void stage_convert(const StageRaw& raw, int m, const Stage<TOK>& st, int s, int lane) {
  constexpr int NT = Stage<TOK>::NT;
  const int q = lane >> 1, jh = (lane & 1) * 4;
  float v[4][4];  // [i][jj]
  float amax = 0.f, tpart = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i][0] = __uint_as_float(raw.x[i].x << 16) * raw.sc[i].x;
    v[i][1] = __uint_as_float(raw.x[i].x & 0xFFFF0000u) * raw.sc[i].y;
    v[i][2] = __uint_as_float(raw.x[i].y << 16) * raw.sc[i].z;
    v[i][3] = __uint_as_float(raw.x[i].y & 0xFFFF0000u) * raw.sc[i].w;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      amax = fmaxf(amax, fabsf(v[i][jj]));
      tpart += v[i][jj];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    tpart += __shfl_xor_sync(0xffffffffu, tpart, o);
  }
  // sigma = 2^sg with max|x'| sigma < 1/2, so that x' sigma 2^9 < 256 <= 448 (e4m3 max).
  const int e = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127 : 0;
  const int sg = max(-126, min(118, -2 - (e < -126 ? -126 : e)));
  const int t = q >> 2, ee = q & 3;
  uint32_t* fr = st.frag_at(s);
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = jh + jj;
    const float f = pow2(sg + 9 - (j & 3));
    float y0 = v[0][jj] * f, y1 = v[1][jj] * f, y2 = v[2][jj] * f, y3 = v[3][jj] * f;
    const int u = j >> 1, half = j & 1;
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) {
      const uint32_t lo = to_e4m3x2(y0, y1), hi = to_e4m3x2(y2, y3);
      const int n = kLimbs * m + l;
      const int nt = n >> 3, gc = n & 7;
      fr[(((ee * 4 + u) * NT + nt) * 32 + 4 * gc + t) * 2 + half] = lo | (hi << 16);
      if (l + 1 < kLimbs) {
        const float2 a = from_e4m3x2(lo), b = from_e4m3x2(hi);
        y0 = (y0 - a.x) * 16.f;
        y1 = (y1 - a.y) * 16.f;
        y2 = (y2 - b.x) * 16.f;
        y3 = (y3 - b.y) * 16.f;
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) st.fcol[s * NT * 8 + kLimbs * m + l] = -2.f * pow2(-sg - 4 * l);
    st.tsb[s * TOK + m] = tpart;
  }
}

// One warp: row tile (rows r0 .. r0+15) x staged super-block slot s, packed words of
// rows g and g+8 (words 4t .. 4t+3 of the super-block) in wg / wh.  Adds the folded
// result into tot.
template <int TOK>
__device__ __forceinline__ void tile_sb(const Stage<TOK>& st, int s, uint4 wg, uint4 wh, float (&tot)[Stage<TOK>::NT][4],
                                        int lane) {
  constexpr int NT = Stage<TOK>::NT;
  const uint32_t* fr = st.frag_at(s);
  float acc[2][NT][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[h][nt][r] = 0.f;
  const uint32_t g4[4] = {wg.x, wg.y, wg.z, wg.w};
  const uint32_t h4[4] = {wh.x, wh.y, wh.z, wh.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t w0 = g4[e], w1 = h4[e];
    const uint32_t x0 = w0 >> 4, x1 = w1 >> 4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t a0 = lanes_of(w0, x0, 2 * u), a1 = lanes_of(w1, x1, 2 * u);
      const uint32_t a2 = lanes_of(w0, x0, 2 * u + 1), a3 = lanes_of(w1, x1, 2 * u + 1);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint2 b = *reinterpret_cast<const uint2*>(fr + (((e * 4 + u) * NT + nt) * 32 + lane) * 2);
        mma_e4m3(acc[e & 1][nt], a0, a1, a2, a3, b.x, b.y);
      }
    }
  }
  const int t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float f0 = st.fcol[s * NT * 8 + 8 * nt + 2 * t], f1 = st.fcol[s * NT * 8 + 8 * nt + 2 * t + 1];
#pragma unroll
    for (int r = 0; r < 4; ++r) tot[nt][r] = fmaf(acc[0][nt][r] + acc[1][nt][r], (r & 1) ? f1 : f0, tot[nt][r]);
  }
}

// Packed words of rows g and g+8 of a row tile for a super-block: words w0 .. w0+3
// where w0 = sb*16 + 4t.  Rows past R and words past Wd read as zero.  kVec: 16-byte
// loads (Wd % 4 == 0 and an aligned base); otherwise four 4-byte loads.
template <bool kVec>
__device__ __forceinline__ uint4 load_words(const uint32_t* S, int64_t R, int64_t Wd, int64_t row, int64_t w0) {
  uint4 r = make_uint4(0u, 0u, 0u, 0u);
  if (row >= R) return r;
  const uint32_t* p = S + row * Wd + w0;
  if constexpr (kVec) {
    if (w0 < Wd) r = __ldcs(reinterpret_cast<const uint4*>(p));
  } else {
    if (w0 + 0 < Wd) r.x = __ldcs(p + 0);
    if (w0 + 1 < Wd) r.y = __ldcs(p + 1);
    if (w0 + 2 < Wd) r.z = __ldcs(p + 2);
    if (w0 + 3 < Wd) r.w = __ldcs(p + 3);
  }
  return r;
}

}  // namespace f8
}  // namespace ob
