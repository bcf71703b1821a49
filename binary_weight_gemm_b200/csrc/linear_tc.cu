// linear_tc.cu -- large-M sign product on the fifth-generation tensor core.
//
//   Y[m, n] = oscale[n] * sum_k x[m, k] * (iscale[k] * s[n, k])
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": [(X ⊙ b^T) W_sign^T] ⊙ a^T,
// computed here with b folded into the sign operand (X ⊙ b^T) S^T = X (S ⊙ 1 b^T)^T;
// "Addition is almost all you need ..." (gist.science), "Methodologie": each of
// DBF's two sign products is one call.
//
// Persistent, warp-specialised kernel, one CTA per SM, output tile 128 weight
// rows x 256 tokens:
//  * warp 12 (one lane): TMA loads of the activation tile (256 tokens x 64 k,
//    bf16, 128-byte swizzle) into a 4-deep shared-memory ring.  This is the MMA's
//    B operand; the activations are never touched by a thread.
//  * warps 0-3: one thread per weight row expands two packed words (64 k) into
//    32 TMEM columns of bf16 pairs (+/-bf16(b_k), +/-bf16(b_k+1)) with
//    tcgen05.st.  This is the MMA's A operand in tensor memory, so the expanded
//    signs cost no shared-memory bandwidth.
//  * warp 13 (one lane): tcgen05.mma kind::f16, M=128, N=256, K=16, fp32
//    accumulators in TMEM (256 columns); tcgen05.commit releases ring slots.
//  * warps 4-11: epilogue, two warps per TMEM lane quadrant (each drains half of
//    the token columns): tcgen05.ld of the accumulator, * oscale, transposed
//    through shared memory into 16-byte stores along Y's rows.
// Every mbarrier wait is bounded (see ob_device.cuh).
#include <algorithm>
#include <cstring>
#include <mutex>

#include <cuda.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kRows = 128;     // MMA M (weight rows)
constexpr int kTok = 256;      // MMA N (tokens)
constexpr int kBK = 64;        // k per stage
constexpr int kMaxStages = 4;
constexpr int kThreads = 448;  // 14 warps
constexpr uint32_t kXStageBytes = kTok * kBK * 2;   // 32 KB
constexpr uint32_t kOutTileBytes = kTok * kRows * 2;  // 64 KB: bf16 output tile staged for the TMA store
constexpr int kTmemCols = 512;                      // D [0,256), A slots 256 + 32*s (s < 4)
constexpr uint32_t kIdesc = idesc_bf16_f32(kRows, kTok);
// iscale pairs live in shared memory (2 bytes per k): four ring stages fit up to
// K = 16384, three up to K = 32768.
constexpr int64_t kMaxK4 = 16384;
constexpr int64_t kMaxK = 32768;
constexpr int kOutDirect = 0, kOutTmaStore = 1, kOutSplit = 2;  // epilogue modes

struct __align__(128) TcShared {  // 128-byte size keeps the bf16x2 table after it 16-byte aligned
  uint64_t full[kMaxStages];   // X tile landed (TMA transaction bytes) and all four A warps stored
  uint64_t empty[kMaxStages];
  uint64_t dfull;
  uint64_t dempty;
  uint64_t stg_full;           // all eight epilogue warps wrote their part of the output tile
  uint64_t stg_free;           // the TMA store has read the output tile
  uint32_t tmem_base;
  int abort_flag;
};

// Separates the even and odd bits of a word: bit j of the result's low half is
// bit 2j of w, bit 16+j is bit 2j+1.  Four exchanges of bit groups (1, 2, 4 and
// 8 bits wide) between neighbouring positions.
__host__ __device__ __forceinline__ uint32_t unzip_bits(uint32_t w) {
  uint32_t t;
  t = (w ^ (w >> 1)) & 0x22222222u; w ^= t ^ (t << 1);
  t = (w ^ (w >> 2)) & 0x0C0C0C0Cu; w ^= t ^ (t << 2);
  t = (w ^ (w >> 4)) & 0x00F000F0u; w ^= t ^ (t << 4);
  t = (w ^ (w >> 8)) & 0x0000FF00u; w ^= t ^ (t << 8);
  return w;
}

__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, unsigned* err, volatile int* abort_flag,
                                          int lane) {
  int okw = 1;
  if (lane == 0) okw = mbar_wait(bar, parity, err, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, okw, 0) != 0;
}

template <int kStages>
__global__ void __launch_bounds__(kThreads, 1) sign_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                                    const __grid_constant__ CUtensorMap tmap_y,
                                                                    SignGemmArgs g, int out_mode, int ksplit,
                                                                    float* part, unsigned* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // [ring: kStages x 32 KB][output tile 64 KB][TcShared][iscale pairs]
  uint8_t* xs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_tile = xs + (size_t)kStages * kXStageBytes;
  TcShared* sh = reinterpret_cast<TcShared*>(out_tile + kOutTileBytes);
  uint32_t* bpair = reinterpret_cast<uint32_t*>(sh + 1);  // [K/2] bf16x2 (iscale[2i], iscale[2i+1])

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t K = g.K, Wd = K / 32;
  const int nkb = (int)((K + kBK - 1) / kBK);
  const int64_t m_blocks = (g.M + kTok - 1) / kTok;
  const int64_t n_blocks = (g.R + kRows - 1) / kRows;
  const int64_t tiles = m_blocks * n_blocks;
  // Work unit u = (tile u / ksplit, k slice u % ksplit).  Slices are whole groups of
  // four stages (8 packed words), so every slice starts 16-byte aligned.
  const int ngroups_k = (nkb + 3) / 4;
  const int64_t units = tiles * ksplit;
  auto unit_k = [&](int64_t u, int& kb0, int& kb1) {
    const int ks = (int)(u % ksplit);
    kb0 = 4 * (int)((int64_t)ks * ngroups_k / ksplit);
    const int end = 4 * (int)((int64_t)(ks + 1) * ngroups_k / ksplit);
    kb1 = end < nkb ? end : nkb;
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 5);  // the TMA thread's expect-tx arrival + one per A warp
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->dfull, 1);
    mbar_init(&sh->dempty, 8);
    mbar_init(&sh->stg_full, 8);
    mbar_init(&sh->stg_free, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  pdl_wait();  // every input may have been written by the previous grid in the stream
  // Input-scale pairs as bf16x2 (round to nearest even); ones without a scale.
  for (int64_t i = tid; i < (K + 1) / 2; i += kThreads) {
    const float lo = g.iscale ? __ldg(g.iscale + 2 * i) : 1.f;
    const float hi = g.iscale ? __ldg(g.iscale + 2 * i + 1) : 1.f;
    bpair[i] = pack_bf16x2(lo, hi);
  }
  if (warp == 13) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort_flag = &sh->abort_flag;
  pdl_launch_dependents();

  if (warp < 4) {
    // ------------------------------------------------ A producer: signs (x) input scale -> TMEM
    // Sign words are fetched a whole group of four stages (8 words) ahead, so an L2
    // round trip is always hidden behind four stages of MMAs.
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const bool vec = (Wd & 3) == 0;
    int64_t gstage = 0;
    bool ok = true;
    // A stage's tcgen05.st is waited for only after the next stage's values are
    // computed: store latency overlaps the expansion arithmetic.
    int pending = -1;
    auto flush_pending = [&]() {
      if (pending >= 0) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->full[pending]);
        pending = -1;
      }
    };
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int64_t tile = u / ksplit;
      int kb0, kb1;
      unit_k(u, kb0, kb1);
      const int64_t n = (tile % n_blocks) * kRows + tid;
      const bool row_ok = n < g.R;
      const uint32_t* srow = g.S + (row_ok ? n : 0) * Wd;
      auto load_group = [&](int64_t grp, uint32_t (&wv)[8]) {
        const int64_t w0 = 2 * (int64_t)kb0 + grp * 8;
        if (vec) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (row_ok && w0 + 4 * h < Wd) v = __ldg(reinterpret_cast<const uint4*>(srow + w0) + h);
            wv[4 * h] = v.x; wv[4 * h + 1] = v.y; wv[4 * h + 2] = v.z; wv[4 * h + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) wv[i] = (row_ok && w0 + i < Wd) ? __ldg(srow + w0 + i) : 0u;
        }
      };
      uint32_t cur[8], nxt[8];
      load_group(0, cur);
      const int ngroups = (kb1 - kb0 + 3) / 4;
      for (int grp = 0; grp < ngroups && ok; ++grp) {
        load_group(grp + 1, nxt);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int kb = kb0 + grp * 4 + i;
          if (kb >= kb1) break;
          const uint32_t w0 = cur[2 * i], w1 = cur[2 * i + 1];
          const uint4* bp = reinterpret_cast<const uint4*>(bpair + (int64_t)kb * (kBK / 2));
          const bool full_stage = (int64_t)(kb + 1) * kBK <= K;
          // Column c of the stage holds k = 2c, 2c+1.  After unzip_bits, bit j of a
          // word's low half is its bit 2j and bit 16+j its bit 2j+1, so one shift
          // puts both signs of a pair on the bf16 sign bits 15 and 31.
          const uint32_t u0 = unzip_bits(w0), u1 = unzip_bits(w1);
          uint32_t v[32];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint4 b4 = make_uint4(0, 0, 0, 0);
            if (full_stage || q < 4) b4 = bp[q];  // a trailing half stage reads 32 k only
            const uint32_t bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = q * 4 + e;
              const uint32_t u = c < 16 ? u0 : u1;
              v[c] = ((u << (15 - (c & 15))) & 0x80008000u) ^ bb[e];
            }
          }
          // The previous stage's store has had this stage's arithmetic to land: only
          // now wait for it and release that stage to the MMA.
          flush_pending();
          const int s = (int)(gstage % kStages);
          if (gstage >= kStages) {
            ok = wait_warp(&sh->empty[s], (uint32_t)((gstage / kStages) - 1) & 1u, err, abort_flag, lane);
            if (!ok) break;
            tc_fence_after();
          }
          tmem_st_x32(lane_base + 256u + 32u * s, v);
          pending = s;
          ++gstage;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
      }
      flush_pending();  // the tile's last stage, before the next tile's sign loads
    }
    flush_pending();
  } else if (warp < 12) {
    // ------------------------------------------------ epilogue
    // Two warps per TMEM lane quadrant; a thread holds one weight row of the
    // accumulator and reads 32 token columns per tcgen05.ld.
    const int q = warp & 3;               // TMEM lane quadrant
    const int half = (warp - 4) >> 2;     // which half of the token columns
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int c0 = half * (kTok / 64), c1 = c0 + kTok / 64;
    int64_t it = 0;
    if (out_mode == kOutSplit) {
      // Split K: this unit's fp32 partial sums, unscaled, to part[k slice][m][n];
      // a second kernel sums the slices and applies the output scale.
      for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
        if (!wait_warp(&sh->dfull, (uint32_t)it & 1u, err, abort_flag, lane)) break;
        tc_fence_after();
        const int64_t tile = u / ksplit, ks = u % ksplit;
        const int64_t m0 = (tile / n_blocks) * kTok;
        const int64_t nr = (tile % n_blocks) * kRows + q * 32 + lane;
        float* dst = part + (ks * g.M) * g.R + nr;
#pragma unroll 1
        for (int c = c0; c < c1; ++c) {
          uint32_t d[32];
          tmem_ld_x32(lane_base + 32u * c, d);
          tmem_wait_ld();
          if (c == c1 - 1) {  // this warp's last read of the accumulator
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->dempty);
          }
          if (nr < g.R) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int64_t m = m0 + 32 * c + i;
              if (m < g.M) dst[m * g.R] = __uint_as_float(d[i]);
            }
          }
        }
      }
    } else if (out_mode == kOutTmaStore) {
      // bf16 Y: the tile is staged in shared memory as [token][row], Y's own
      // layout, and written by one TMA store that clips the ragged edges.  The
      // accumulator is released right after its last tcgen05.ld, so the next
      // tile's MMAs overlap the conversion and the store.
      uint16_t* col = reinterpret_cast<uint16_t*>(out_tile) + q * 32 + lane;
      for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {  // ksplit == 1
        if (!wait_warp(&sh->dfull, (uint32_t)it & 1u, err, abort_flag, lane)) break;
        tc_fence_after();
        if (it > 0 && !wait_warp(&sh->stg_free, (uint32_t)(it - 1) & 1u, err, abort_flag, lane)) break;
        const int64_t m0 = (tile / n_blocks) * kTok;
        const int64_t n0 = (tile % n_blocks) * kRows;
        const int64_t nr = n0 + q * 32 + lane;
        const float sc = nr < g.R ? __ldg(g.oscale + nr) : 0.f;
#pragma unroll 1
        for (int c = c0; c < c1; ++c) {
          uint32_t d[32];
          tmem_ld_x32(lane_base + 32u * c, d);
          tmem_wait_ld();
          if (c == c1 - 1) {  // this warp's last read of the accumulator
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh->dempty);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i)
            col[(32 * c + i) * kRows] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(d[i]) * sc));
        }
        fence_proxy_async_smem();  // the tile is read by the TMA (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->stg_full);
        if (warp == 4 && lane == 0) {
          if (mbar_wait(&sh->stg_full, (uint32_t)it & 1u, err, abort_flag)) {
            tma_store_2d(&tmap_y, out_tile, (int32_t)n0, (int32_t)m0);
            bulk_commit_group();
            bulk_wait_read_all();
          }
          mbar_arrive(&sh->stg_free);
        }
        __syncwarp();
      }
      if (warp == 4 && lane == 0) bulk_wait_all();
    } else {
      // fp32 Y, or a Y the TMA cannot address: each warp transposes its 32 x 32
      // blocks through shared memory so that every store is a 16-byte piece of
      // one Y row (8 bf16 or 4 fp32 consecutive outputs).
      float* scr = reinterpret_cast<float*>(out_tile) + (warp - 4) * (32 * 33);
      const bool f32 = g.y_dtype == OB_OUT_F32;
      const bool vec_ok = (g.ldy % (f32 ? 4 : 8)) == 0 && (reinterpret_cast<uintptr_t>(g.Y) & 15) == 0;
      for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {  // ksplit == 1
        if (!wait_warp(&sh->dfull, (uint32_t)it & 1u, err, abort_flag, lane)) break;
        tc_fence_after();
        const int64_t m0 = (tile / n_blocks) * kTok;
        const int64_t nq = (tile % n_blocks) * kRows + q * 32;  // this warp's 32 weight rows
        const float sc = (nq + lane < g.R) ? __ldg(g.oscale + nq + lane) : 0.f;
#pragma unroll 1
        for (int c = c0; c < c1; ++c) {
          uint32_t d[32];
          tmem_ld_x32(lane_base + 32u * c, d);
          tmem_wait_ld();
          // scr[token][row], row = lane (pitch 33 floats: conflict-free both ways)
#pragma unroll
          for (int i = 0; i < 32; ++i) scr[i * 33 + lane] = __uint_as_float(d[i]) * sc;
          __syncwarp();
          const int64_t mc = m0 + 32 * c;
          if (f32) {
            // 32 tokens x 8 pieces of 4 outputs: lane -> (token, piece)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int v = lane + 32 * i, tok = v >> 3, pc = v & 7;
              const int64_t m = mc + tok, n = nq + 4 * pc;
              if (m < g.M) {
                const float* src = scr + tok * 33 + 4 * pc;
                float* dst = static_cast<float*>(g.Y) + m * g.ldy + n;
                if (vec_ok && n + 4 <= g.R) {
                  *reinterpret_cast<float4*>(dst) = make_float4(src[0], src[1], src[2], src[3]);
                } else {
                  for (int e = 0; e < 4; ++e)
                    if (n + e < g.R) dst[e] = src[e];
                }
              }
            }
          } else {
            // 32 tokens x 4 pieces of 8 outputs
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int v = lane + 32 * i, tok = v >> 2, pc = v & 3;
              const int64_t m = mc + tok, n = nq + 8 * pc;
              if (m < g.M) {
                const float* src = scr + tok * 33 + 8 * pc;
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(g.Y) + m * g.ldy + n;
                if (vec_ok && n + 8 <= g.R) {
                  uint4 o;
                  o.x = pack_bf16x2(src[0], src[1]); o.y = pack_bf16x2(src[2], src[3]);
                  o.z = pack_bf16x2(src[4], src[5]); o.w = pack_bf16x2(src[6], src[7]);
                  *reinterpret_cast<uint4*>(dst) = o;
                } else {
                  for (int e = 0; e < 8; ++e)
                    if (n + e < g.R) dst[e] = __float2bfloat16_rn(src[e]);
                }
              }
            }
          }
          __syncwarp();  // scr is rewritten by the next chunk
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->dempty);
      }
    }
  } else if (warp == 12) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
        int64_t gstage = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int32_t m0 = (int32_t)((u / ksplit / n_blocks) * kTok);
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++gstage) {
          const int s = (int)(gstage % kStages);
          if (gstage >= kStages) {
            ok = mbar_wait(&sh->empty[s], (uint32_t)((gstage / kStages) - 1) & 1u, err, abort_flag);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(&sh->full[s], kXStageBytes);
          tma_load_2d(xs + (size_t)s * kXStageBytes, &tmap_x, &sh->full[s], kb * kBK, m0);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors of ring slot 0; slot s adds s * kXStageBytes to the start
      // address field (address >> 4, no carry out of its 14 bits below 256 KB).
      const uint32_t xa0 = smem_u32(xs);
      const uint64_t d0 = sdesc_kmajor_sw128(xa0), d1 = sdesc_kmajor_sw128(xa0 + 32u);
      const uint64_t d2 = sdesc_kmajor_sw128(xa0 + 64u), d3 = sdesc_kmajor_sw128(xa0 + 96u);
      uint32_t s = 0, phase = 0;
      int64_t it = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x, ++it) {
        if (it > 0) {
          ok = mbar_wait(&sh->dempty, (uint32_t)(it - 1) & 1u, err, abort_flag);
          if (!ok) break;
          tc_fence_after();
        }
        int kb0, kb1;
        unit_k(u, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          // One barrier per stage for both operands: a second wait costs the issuing
          // thread about a hundred cycles per stage.
          ok = mbar_wait(&sh->full[s], phase, err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          // The four descriptors are ready before the first MMA of the stage, each in
          // its own register, and the MMAs are unrolled: an MMA reads its operand
          // registers after issue, so rewriting them for the next MMA would stall.
          const uint64_t so = (uint64_t)(s * (kXStageBytes >> 4));
          const uint64_t b0 = d0 + so, b1 = d1 + so, b2 = d2 + so, b3 = d3 + so;
          const uint32_t aa = tmem + 256u + 32u * s;
          mma_bf16_ts(tmem, aa, b0, kIdesc, kb > kb0 ? 1u : 0u);
          mma_bf16_ts(tmem, aa + 8u, b1, kIdesc, 1u);
          if ((int64_t)(kb + 1) * kBK <= K) {  // a trailing half stage holds 32 k
            mma_bf16_ts(tmem, aa + 16u, b2, kIdesc, 1u);
            mma_bf16_ts(tmem, aa + 24u, b3, kIdesc, 1u);
          }
          mma_commit(&sh->empty[s]);
          if (++s == (uint32_t)kStages) {
            s = 0;
            phase ^= 1u;
          }
        }
        mma_commit(&sh->dfull);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host: tensor map

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

int64_t sign_gemm_tc_max_k() { return kMaxK; }

void* tensor_map_encode_tiled_fn() { return reinterpret_cast<void*>(get_encode_fn()); }

int tc_split_k(int64_t M, int64_t R, int64_t K, int num_sms) {
  const int64_t tiles = ((M + kTok - 1) / kTok) * ((R + kRows - 1) / kRows);
  if (tiles == 0 || tiles * 2 > num_sms) return 1;
  // K slices are whole 4-stage groups, and at least 16 stages (1024 k) long: shorter
  // slices cost more in the extra partial-sum pass than they gain (measured on B200).
  const int64_t nkb = (K + kBK - 1) / kBK;
  const int64_t ks = std::min<int64_t>(std::min<int64_t>(8, num_sms / tiles), std::min<int64_t>((nkb + 3) / 4, nkb / 16));
  return ks > 1 ? (int)ks : 1;
}

namespace {

// Y[m, n] = oscale[n] * sum over k slices of part[slice][m][n]; 4 consecutive n per item.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* part, int ksplit, int64_t M, int64_t R,
                                                            const float* oscale, void* Y, int64_t ldy, int y_dtype) {
  pdl_wait();  // the partial sums come from the previous grid
  pdl_launch_dependents();
  const int64_t r4 = R / 4, items = M * r4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < items; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / r4, n = (i - m * r4) * 4;
    float4 acc = __ldcg(reinterpret_cast<const float4*>(part + m * R + n));
    for (int ks = 1; ks < ksplit; ++ks) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(part + ((int64_t)ks * M + m) * R + n));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const float4 sc = __ldg(reinterpret_cast<const float4*>(oscale + n));
    acc.x *= sc.x; acc.y *= sc.y; acc.z *= sc.z; acc.w *= sc.w;
    if (y_dtype == OB_OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(Y) + m * ldy + n) = acc;
    } else {
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(Y) + m * ldy + n) =
          make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
  }
}

cudaError_t launch_tc_impl(const SignGemmArgs& g, int ksplit, float* part, const LaunchCtx& c) {
  if (g.M == 0 || g.R == 0 || g.K == 0) return cudaSuccess;
  if (g.K > kMaxK) return cudaErrorInvalidValue;
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return cudaErrorNotSupported;

  CUtensorMap tmap_x, tmap_y;
  std::memset(&tmap_x, 0, sizeof(tmap_x));
  std::memset(&tmap_y, 0, sizeof(tmap_y));
  {
    const cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.M};
    const cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kTok};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(g.X), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  // bf16 Y whose rows start on 16-byte boundaries is written by TMA stores.
  int tma_store = 0;
  if (ksplit == 1 && g.y_dtype == OB_OUT_BF16 && g.ldy % 8 == 0 && (reinterpret_cast<uintptr_t>(g.Y) & 15) == 0) {
    const cuuint64_t dims[2] = {(cuuint64_t)g.R, (cuuint64_t)g.M};
    const cuuint64_t strides[1] = {(cuuint64_t)g.ldy * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRows, (cuuint32_t)kTok};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tmap_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.Y, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    tma_store = r == CUDA_SUCCESS ? 1 : 0;
  }

  const int64_t tiles = ((g.M + kTok - 1) / kTok) * ((g.R + kRows - 1) / kRows);
  const int grid = (int)std::min<int64_t>(tiles * ksplit, c.num_sms);
  const int out_mode = ksplit > 1 ? kOutSplit : (tma_store ? kOutTmaStore : kOutDirect);
  const int stages = g.K <= kMaxK4 ? 4 : 3;
  const size_t smem = 1024 + (size_t)stages * kXStageBytes + kOutTileBytes + sizeof(TcShared) +
                      sizeof(uint32_t) * ((((g.K + 1) / 2) + 3) & ~int64_t(3));

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (c.pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    na = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  auto kern = stages == 4 ? sign_gemm_tc_kernel<4> : sign_gemm_tc_kernel<3>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, kern, tmap_x, tmap_y, g, out_mode, ksplit, part, c.err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sign_gemm_tc(const SignGemmArgs& g, const LaunchCtx& c) { return launch_tc_impl(g, 1, nullptr, c); }

cudaError_t launch_sign_gemm_tc_splitk(const SignGemmArgs& g, int ksplit, float* part, const LaunchCtx& c) {
  if (g.M == 0 || g.R == 0 || g.K == 0) return cudaSuccess;
  // The same limits as tc_split_k: whole 4-stage groups of at least 16 stages.
  const int64_t nkb = (g.K + kBK - 1) / kBK;
  ksplit = (int)std::min<int64_t>(ksplit, std::min<int64_t>((nkb + 3) / 4, nkb / 16));
  if (ksplit <= 1 || g.R % 4 != 0 || g.ldy % 4 != 0) return launch_tc_impl(g, 1, nullptr, c);
  cudaError_t e = launch_tc_impl(g, ksplit, part, c);
  if (e != cudaSuccess) return e;
  const int64_t items = g.M * (g.R / 4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min<int64_t>((items + 255) / 256, (int64_t)c.num_sms * 8), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, static_cast<const float*>(part), ksplit, g.M, g.R, g.oscale,
                         g.Y, g.ldy, g.y_dtype);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ob
