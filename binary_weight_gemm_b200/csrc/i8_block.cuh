// i8_block.cuh -- the sign product on int8 tensor cores: packed signs become u8 operands
// with one AND per four weights.
//
//   Y[m, n] = oscale[n] * sum_k x'[m, k] s[n, k],   x' = x ⊙ iscale,  s = 1 - 2 bit
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T;
// "Addition is almost all you need ..." (gist.science), "Methodologie": a product with
// a +/-1 matrix needs no multiplications.  The tensor core does the additions; what is
// minimised is the cost of getting the packed signs into its operand format.
//
// Identity used: sum_k s_k x'_k = T - 2 sum_k bit_k x'_k, with T = sum_k x'_k.  The masked
// sum is an exact integer dot product, computed by mma.sync.m16n8k32 with u8 x s8 -> s32
// (native on sm_100a: e4m3 and 4-bit forms measured three to twenty times slower with
// operands that change every instruction):
//
//  * x' is quantised per token and per super-block of 512 k: q = rint(x' sigma) with a
//    power-of-two sigma such that |q| <= 2^20, and split into three base-128 limbs
//    q = l0 + 128 l1 + 16384 l2 (l0, l1 in [0, 128), l2 in [-64, 64]).  Column n = 3 m + l of
//    the B operand holds limb l of token m.  The rounding is the only approximation (2^-21
//    of the super-block's largest |x'|); one warp stages a (token, super-block) pair on its
//    own, scale included.
//  * A (16 rows x 32 k, weights): for bit position j = 2i + c (i = 0..3, c = 0, 1) the
//    register (w >> 2i) & (0x01010101 << c) of a packed word w holds, in byte i', bit
//    8i' + j of w at bit c: the u8 value 2^c bit (one shift per word and i, one AND per
//    four weights).  One MMA takes a single position j from two packed words (a0/a1 from
//    word 2p, a2/a3 from word 2p+1 of the lane's four) and accumulates into chain (p, c):
//    four chains, whose sum of acc >> c is the exact integer sum of bit * limb.
//  * The integer sums of a (tile, super-block) are converted and scaled, -2 * 128^l / sigma
//    per column; T is added in the epilogue.
//
// Fragment correspondence (PTX ISA, mma.m16n8k32 with 8-bit operands): lane (g, t) holds
// A rows g and g+8, k-slots 4t + i (a0, a1) and 16 + 4t + i (a2, a3), and B column g,
// k-slots 4t + i (b0) and 16 + 4t + i (b1).  A super-block is 512 k = 16 packed words per
// row; lane t of a quad owns words 4t .. 4t+3 (one 16-byte load per row).  MMA (p, j) of
// a super-block (p = 0, 1; j = 0..7) maps k-slot 4t + i to k = 32 (4t + 2p) + 8i + j and
// k-slot 16 + 4t + i to k = 32 (4t + 2p + 1) + 8i + j.  The B fragments are staged in
// shared memory in that order, [p][j][lane] as uint2 (b0, b1).
#pragma once

#include <cuda_bf16.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace i8 {

constexpr int kLimbs = 3;
constexpr int kSbK = 512;                    // k per super-block
constexpr int kSbWords = kSbK / 32;          // packed words per row per super-block
constexpr int kFragWords = 2 * 8 * 32 * 2;   // 32-bit words of B fragments per super-block
constexpr int kMaxTok = 2;                   // tokens per pass: 3 limbs x 2 tokens fill one n8 tile

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// Shared-memory layout of a staged chunk of `ch` super-blocks for TOK <= 2 tokens.
template <int TOK>
struct Stage {
  uint32_t* frag;  // [ch][p][j][lane][2]
  float* fsb;      // [ch][8]: fold factor of each accumulator column for the super-block
  float* tsb;      // [ch][TOK]: sum of x' over the super-block, per token
  __device__ __forceinline__ uint32_t* frag_at(int s) const { return frag + (size_t)s * kFragWords; }
  __device__ __forceinline__ const float* fold_at(int s) const { return fsb + (size_t)s * 8; }
  static __host__ __device__ constexpr size_t bytes_per_sb() {
    return sizeof(uint32_t) * kFragWords + sizeof(float) * (8 + TOK);
  }
  static __host__ __device__ constexpr size_t bytes(int ch) { return bytes_per_sb() * (size_t)ch; }
  __device__ static Stage carve(uint8_t* base, int ch) {
    Stage st;
    st.frag = reinterpret_cast<uint32_t*>(base);
    st.fsb = reinterpret_cast<float*>(base + sizeof(uint32_t) * (size_t)ch * kFragWords);
    st.tsb = st.fsb + (size_t)ch * 8;
    return st;
  }
};

// The raw inputs one lane needs for a (token, super-block) pair: x (bf16) and the input
// scale at k = kbase + 32 q + 8 i + j, q = lane / 2, j = 4 (lane & 1) .. + 3, i = 0..3.
struct StageRaw {
  uint2 x[4];
  float4 sc[4];
};

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

// Stage a pair from tagged words instead of X: word k of token m is kTagMark | bf16 bits at
// tags[m * K + k], written by an earlier layer of the same launch.  Loads the lane's words
// (relaxed, from L2) and its input scales into r; returns whether all of the lane's words
// carry the mark (words past K or of a token not present count as ready).
__device__ __forceinline__ bool stage_load_tagged(const SignGemmArgs& g, const uint32_t* tags, int64_t m_glob,
                                                  bool live, int64_t kbase, int lane, StageRaw& r) {
  const int q = lane >> 1, jh = (lane & 1) * 4;
  const int64_t K = g.K;
  bool ready = true;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k0 = kbase + 32 * q + 8 * i + jh;
    r.sc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    r.x[i] = make_uint2(0u, 0u);
    if (live && k0 < K) {
      r.sc[i] = g.iscale ? __ldg(reinterpret_cast<const float4*>(g.iscale + k0)) : make_float4(1.f, 1.f, 1.f, 1.f);
      const uint4 w = ld_volatile_v4(tags + m_glob * K + k0);
      ready &= ((w.x & w.y & w.z & w.w) >> 16) == (kTagMark >> 16) && ((w.x | w.y | w.z | w.w) >> 16) == (kTagMark >> 16);
      r.x[i] = make_uint2(__byte_perm(w.x, w.y, 0x5410), __byte_perm(w.z, w.w, 0x5410));
    }
  }
  return ready;
}

// x' of the lane's 16 values: v[i][jj] at k = kbase + 32 q + 8 i + jh + jj.
__device__ __forceinline__ void stage_values(const StageRaw& raw, float (&v)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i][0] = __uint_as_float(raw.x[i].x << 16) * raw.sc[i].x;
    v[i][1] = __uint_as_float(raw.x[i].x & 0xFFFF0000u) * raw.sc[i].y;
    v[i][2] = __uint_as_float(raw.x[i].y << 16) * raw.sc[i].z;
    v[i][3] = __uint_as_float(raw.x[i].y & 0xFFFF0000u) * raw.sc[i].w;
  }
}

// q = rint(y) for |y| < 2^22, by the float magic-number rounding (one FFMA, one integer
// subtract: round to nearest even, as the FFMA rounds).
__device__ __forceinline__ int rint_small(float v, float sigma) {
  return __float_as_int(fmaf(v, sigma, 12582912.f)) - 0x4B400000;  // 12582912 = 1.5 * 2^23
}

// The three limbs of four values q0..q3 (|q| <= 2^20) as s8 registers, byte i from q_i:
// q = l0 + 128 l1 + 16384 l2 with l0, l1 in [0, 128) and l2 = q >> 14 in [-64, 64].
// l0 is byte 0 of q masked to 7 bits, l1 byte 1 of 2q masked, l2 byte 2 of 4q (the bits
// above are copies of the sign for |q| <= 2^20, so the byte is l2 in two's complement).
__device__ __forceinline__ void limb_regs(int q0, int q1, int q2, int q3, uint32_t (&reg)[3]) {
  const uint32_t a0 = q0, a1 = q1, a2 = q2, a3 = q3;
  reg[0] = __byte_perm(__byte_perm(a0, a1, 0x0040), __byte_perm(a2, a3, 0x0040), 0x5410) & 0x7F7F7F7Fu;
  const uint32_t d0 = a0 << 1, d1 = a1 << 1, d2 = a2 << 1, d3 = a3 << 1;
  reg[1] = __byte_perm(__byte_perm(d0, d1, 0x0051), __byte_perm(d2, d3, 0x0051), 0x5410) & 0x7F7F7F7Fu;
  const uint32_t f0 = a0 << 2, f1 = a1 << 2, f2 = a2 << 2, f3 = a3 << 2;
  reg[2] = __byte_perm(__byte_perm(f0, f1, 0x0062), __byte_perm(f2, f3, 0x0062), 0x5410);
}

// Stage a (token m, super-block s) pair into slot s: the pair's largest |x'| gives its scale
// sigma = 2^sg (max |x'| sigma < 2^20), its limbs go to the B fragments, its fold factors
// (-2 * 128^l / sigma for columns 3 m + l; the warp of token 0 also zeroes the unused
// columns) and its sum of x' to the slot's tables.  All lanes of a warp call it.
template <int TOK>
__device__ __forceinline__ void stage_pair(const StageRaw& raw, int m, const Stage<TOK>& st, int s, int lane) {
  float v[4][4];
  stage_values(raw, v);
  float amax = 0.f, tpart = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      amax = fmaxf(amax, fabsf(v[i][jj]));
      tpart += v[i][jj];
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    tpart += __shfl_xor_sync(0xffffffffu, tpart, o);
  }
  // sigma = 2^sg with sg = 19 - e keeps max |q| < 2^20; sg in [-108, 126] keeps sigma and the
  // fold factors 2^(1 + 7 l - sg) normal floats.  Only a pair whose largest |x'| is below
  // 2^-107 (sub-normal range) keeps fewer than 20 bits.
  const int e = amax > 0.f ? (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127 : 0;
  const int sg = max(-108, min(126, 19 - (e < -126 ? -126 : e)));
  const int q = lane >> 1, jh = (lane & 1) * 4;
  const int t = q >> 2, ee = q & 3, p = ee >> 1, half = ee & 1;
  const float sigma = pow2(sg);
  uint32_t* fr = st.frag_at(s);
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = jh + jj;
    uint32_t reg[kLimbs];
    limb_regs(rint_small(v[0][jj], sigma), rint_small(v[1][jj], sigma), rint_small(v[2][jj], sigma),
              rint_small(v[3][jj], sigma), reg);
#pragma unroll
    for (int l = 0; l < kLimbs; ++l) {
      const int gc = kLimbs * m + l;  // B column (one n8 tile: TOK <= 2)
      fr[((p * 8 + j) * 32 + 4 * gc + t) * 2 + half] = reg[l];
    }
  }
  float* f = st.fsb + (size_t)s * 8;
  if (lane < kLimbs) f[kLimbs * m + lane] = -2.f * pow2(7 * lane - sg);
  if (m == 0 && lane >= kLimbs * TOK && lane < 8) f[lane] = 0.f;
  if (lane == 0) st.tsb[s * TOK + m] = tpart;
}

// Chains per tile: (p, c) with p the word pair and c the parity of the bit position.
constexpr int kChains = 4;

// The A registers of bit position j = 2i + c from the shifted words (word >> 2i).
__device__ __forceinline__ void mma_pos(int (&acc)[4], uint32_t g0, uint32_t h0, uint32_t g1, uint32_t h1, int c,
                                        uint2 b) {
  const uint32_t msk = 0x01010101u << c;
  mma_u8s8(acc, g0 & msk, h0 & msk, g1 & msk, h1 & msk, b.x, b.y);
}

// One tile's rows g / g+8 (packed words wg / wh: words 4t .. 4t+3 of the super-block)
// times staged super-block s, accumulated into the four chains.
__device__ __forceinline__ void tile_sb(const uint32_t* fr, uint4 wg, uint4 wh, int (&acc)[kChains][4], int lane) {
  const uint32_t g4[4] = {wg.x, wg.y, wg.z, wg.w};
  const uint32_t h4[4] = {wh.x, wh.y, wh.z, wh.w};
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t g0 = g4[2 * p] >> (2 * i), h0 = h4[2 * p] >> (2 * i);
      const uint32_t g1 = g4[2 * p + 1] >> (2 * i), h1 = h4[2 * p + 1] >> (2 * i);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int j = 2 * i + c;
        const uint2 b = *reinterpret_cast<const uint2*>(fr + ((p * 8 + j) * 32 + lane) * 2);
        mma_pos(acc[2 * p + c], g0, h0, g1, h1, c, b);
      }
    }
}

// The B fragments of one staged super-block in registers, for a warp that applies one
// super-block to several tiles.
struct SbRegs {
  uint2 b[2][8];
};

__device__ __forceinline__ void load_sb_regs(const uint32_t* fr, int lane, SbRegs& r) {
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int j = 0; j < 8; ++j) r.b[p][j] = *reinterpret_cast<const uint2*>(fr + ((p * 8 + j) * 32 + lane) * 2);
}

// tile_sb with the super-block's fragments already in registers.
__device__ __forceinline__ void tile_sb_regs(const SbRegs& fr, uint4 wg, uint4 wh, int (&acc)[kChains][4]) {
  const uint32_t g4[4] = {wg.x, wg.y, wg.z, wg.w};
  const uint32_t h4[4] = {wh.x, wh.y, wh.z, wh.w};
  // Position-major order: the four chains take turns, so consecutive MMAs never depend on
  // each other.
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const uint32_t g0 = g4[2 * p] >> (2 * i), h0 = h4[2 * p] >> (2 * i);
      const uint32_t g1 = g4[2 * p + 1] >> (2 * i), h1 = h4[2 * p + 1] >> (2 * i);
#pragma unroll
      for (int c = 0; c < 2; ++c) mma_pos(acc[2 * p + c], g0, h0, g1, h1, c, fr.b[p][2 * i + c]);
    }
}

// sum over the chains of acc >> c for accumulator register r: the exact integer sum of
// bit * limb.
__device__ __forceinline__ int combine(const int (&acc)[kChains][4], int r) {
  return (acc[0][r] + acc[2][r]) + ((acc[1][r] + acc[3][r]) >> 1);
}

// Packed words of rows g / g+8 of a row tile for a super-block, from global memory: words
// w0 .. w0+3 of `row`.  Rows past R and words past Wd read as zero.  kVec: one 16-byte load
// (Wd % 4 == 0 and an aligned base); otherwise four 4-byte loads.
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

// The sum of x' over the chunk's chn super-blocks for token m (all lanes of a warp call it;
// the same fixed order on every call: lane s sums super-blocks s, s + 32, ..., then a
// butterfly over the lanes).
template <int TOK>
__device__ __forceinline__ float chunk_sum(const Stage<TOK>& st, int chn, int m, int lane) {
  float t = 0.f;
  for (int s = lane; s < chn; s += 32) t += st.tsb[s * TOK + m];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

}  // namespace i8
}  // namespace ob
