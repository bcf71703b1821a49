// linear_tc2.cu -- large-M sign product on a CTA pair (tcgen05 cta_group::2).
//
//   Y[m, n] = oscale[n] * sum_k x[m, k] * (iscale[k] * s[n, k])
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": [(X ⊙ b^T) W_sign^T] ⊙ a^T, with
// b folded into the sign operand as in linear_tc.cu.
//
// The same warp roles as linear_tc.cu, on a 2-CTA cluster that computes a 256 weight
// rows x kTok tokens tile (kTok = 256, or 128 when the output has few tiles) with
// M = 256 MMAs issued by rank 0:
//  * each CTA expands its own 128 weight rows into its TMEM (rows 0..127 of the MMA's
//    A in rank 0, 128..255 in rank 1) and loads its own kTok / 2 tokens of the
//    activation tile (half of the MMA's N) by TMA, so per SM the activation traffic from
//    L2 and the shared-memory reads of the MMA are half those of the one-CTA kernel;
//  * a stage holds 128 k (two 64-k slabs of 128-byte-swizzled rows), 8 MMAs of
//    256 x kTok x 16, so the per-stage hand-off is amortised over more math;
//  * rank 0's `full` barrier receives both CTAs' TMA bytes and the arrivals of both
//    CTAs' expansion warps; the MMA thread's commits arrive on the `empty` / `dfull`
//    barriers of both CTAs; both epilogues release the accumulator on rank 0's
//    `dempty`.  No load is multicast.
// Every mbarrier wait is bounded; the pair meets at cluster barriers only at the
// start (after barrier setup and TMEM allocation) and at the end (before freeing
// TMEM), which every thread reaches.
#include <algorithm>
#include <cstring>

#include <cuda.h>
#include <cuda_bf16.h>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kRowsCta = 128;   // weight rows per CTA (MMA M = 256 per pair)
constexpr int kBK = 128;        // k per stage
constexpr int kThreads = 448;   // 14 warps
constexpr int kTmemCols = 512;  // D [0, kTok), A slots kTok + 64*s
constexpr int64_t kMaxK = 16384;
// Warp roles: 0-7 expand signs (two per TMEM lane quadrant, each half of a stage's
// 64 columns), 8-11 epilogue (one per quadrant), 12 TMA, 13 MMA (rank 0) + TMEM.
constexpr int kAWarps = 8, kEpiWarps = 4, kEpiWarp0 = 8, kTmaWarp = 12, kMmaWarp = 13;

// Tile shapes: kTok tokens per pair tile (MMA N), 256 or 128.  The narrow tile doubles
// the number of tiles of an output with few of them (e.g. M = 512); its accumulator
// takes 128 TMEM columns, which leaves room for six A stages instead of four.
template <int kTok>
struct Tc2Shape {
  static constexpr int kTokCta = kTok / 2;                         // tokens loaded by each CTA
  static constexpr int kStages = kTok == 256 ? 4 : 6;
  static constexpr uint32_t kSlabBytes = kTokCta * 64 * 2;         // kTokCta tokens x 64 k
  static constexpr uint32_t kStageBytes = 2 * kSlabBytes;          // per CTA
  static constexpr uint32_t kOutTileBytes = kTok * kRowsCta * 2;   // bf16 output tile
  static constexpr uint32_t kASlot0 = kTok;                        // TMEM column of A slot 0
  static constexpr uint32_t kIdesc = idesc_bf16_f32(2 * kRowsCta, kTok);
  static_assert(kTok == 256 || kTok == 128, "pair tile of 256 or 128 tokens");
  static_assert(kASlot0 + 64 * kStages <= kTmemCols, "accumulator and A stages fit TMEM");
};

template <int kStages>
struct __align__(128) Tc2Shared {
  uint64_t full[kStages];  // rank 0: both CTAs' TMA bytes + 8 expansion warps + rank 0's TMA arrival
  uint64_t empty[kStages];  // both CTAs: the pair commit
  uint64_t dfull;           // both CTAs: the pair commit after a tile's last MMA
  uint64_t dempty;          // rank 0: the 16 epilogue warps of the pair
  uint64_t stg_full;        // this CTA's 8 epilogue warps wrote the output tile
  uint64_t stg_free;        // the TMA store has read it
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, unsigned* err, volatile int* abort_flag,
                                          int lane) {
  int okw = 1;
  if (lane == 0) okw = mbar_wait_sleep(bar, parity, err, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, okw, 0) != 0;
}

__host__ __device__ __forceinline__ uint32_t unzip_bits2(uint32_t w) {
  uint32_t t;
  t = (w ^ (w >> 1)) & 0x22222222u; w ^= t ^ (t << 1);
  t = (w ^ (w >> 2)) & 0x0C0C0C0Cu; w ^= t ^ (t << 2);
  t = (w ^ (w >> 4)) & 0x00F000F0u; w ^= t ^ (t << 4);
  t = (w ^ (w >> 8)) & 0x0000FF00u; w ^= t ^ (t << 8);
  return w;
}

// The 32 TMEM columns of one half stage (64 k) of one weight row: column c holds the
// bf16x2 pair of k = 2c, 2c+1, the two signs (from the unzipped words: u0 for columns
// 0..15, u1 for 16..31) on the sign bits of bf16x2(iscale[k], iscale[k+1]) from bp.
// kTail: a trailing partial stage; columns at or past `valid` (counted from the stage's
// first column; this half starts at cbase0) are zero.
template <bool kTail>
__device__ __forceinline__ void expand_half(uint32_t u0, uint32_t u1, const uint4* bp, int cbase0, int valid,
                                            uint32_t (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int cbase = cbase0 + 4 * q;
    uint4 b4 = make_uint4(0, 0, 0, 0);
    if (!kTail || cbase < valid) b4 = bp[q];
    const uint32_t bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 4 * q + e;  // column within this half
      const uint32_t u = c < 16 ? u0 : u1;
      const uint32_t x = ((u << (15 - (c & 15))) & 0x80008000u) ^ bb[e];
      v[c] = (!kTail || cbase + e < valid) ? x : 0u;
    }
  }
}

template <int kTok>
__global__ void __launch_bounds__(kThreads, 1) sign_gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                                     const __grid_constant__ CUtensorMap tmap_y,
                                                                     SignGemmArgs g, unsigned* err) {
  using Sh = Tc2Shape<kTok>;
  constexpr int kTokCta = Sh::kTokCta, kStages = Sh::kStages;
  constexpr uint32_t kSlabBytes = Sh::kSlabBytes, kStageBytes = Sh::kStageBytes, kASlot0 = Sh::kASlot0;
  using Shared = Tc2Shared<kStages>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // [ring: kStages x kStageBytes][output tile][Shared][iscale pairs]; the same offsets in
  // both CTAs (the MMA reads B at one offset in each).
  uint8_t* xs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_tile = xs + (size_t)kStages * kStageBytes;
  Shared* sh = reinterpret_cast<Shared*>(out_tile + Sh::kOutTileBytes);
  uint32_t* bpair = reinterpret_cast<uint32_t*>(sh + 1);  // [K/2] bf16x2 (iscale[2i], iscale[2i+1])

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int64_t pair = cluster_id_x(), npairs = num_clusters_x();
  const int64_t K = g.K, Wd = K / 32;
  const int nkb = (int)((K + kBK - 1) / kBK);
  const int64_t m_blocks = (g.M + kTok - 1) / kTok;
  const int64_t n_blocks = (g.R + 2 * kRowsCta - 1) / (2 * kRowsCta);
  const int64_t tiles = m_blocks * n_blocks;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1 + 2 * kAWarps);  // rank 0's TMA arrival + both CTAs' A warps
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->dfull, 1);
    mbar_init(&sh->dempty, 2 * kEpiWarps);
    mbar_init(&sh->stg_full, kEpiWarps);
    mbar_init(&sh->stg_free, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  pdl_wait();  // every input may have been written by the previous grid in the stream
  for (int64_t i = tid; i < (K + 1) / 2; i += kThreads) {
    const float lo = g.iscale ? __ldg(g.iscale + 2 * i) : 1.f;
    const float hi = g.iscale ? __ldg(g.iscale + 2 * i + 1) : 1.f;
    bpair[i] = pack_bf16x2(lo, hi);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(&sh->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort_flag = &sh->abort_flag;
  pdl_launch_dependents();
  // Rank 0's barriers as cluster addresses (used by both CTAs).
  const uint32_t full0 = mapa_shared(&sh->full[0], 0);
  const uint32_t dempty0 = mapa_shared(&sh->dempty, 0);

  if (warp < kAWarps) {
    // ------------------------------------------------ A producer: this CTA's 128 weight rows
    // Warp w: TMEM lane quadrant w % 4 (32 rows), column half w / 4 of each stage
    // (32 columns = two packed words = 64 k).
    const int aq = warp & 3, ahalf = warp >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(aq * 32) << 16);
    const bool vec = (Wd & 3) == 0;
    int64_t gstage = 0;
    bool ok = true;
    // A stage's TMEM store is waited for (and the stage released to the MMA on rank 0's
    // `full` barrier) only after the next stage's columns are computed, so the store's
    // latency overlaps that arithmetic.
    int pending = -1;
    auto flush_pending = [&]() {
      if (pending >= 0) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(full0 + 8u * pending);
        pending = -1;
      }
    };
    for (int64_t tile = pair; tile < tiles && ok; tile += npairs) {
      const int64_t n = (tile % n_blocks) * (2 * kRowsCta) + rank * kRowsCta + aq * 32 + lane;
      const bool row_ok = n < g.R;
      const uint32_t* srow = g.S + (row_ok ? n : 0) * Wd;
      // 8 words = two stages, fetched a group ahead.
      auto load_group = [&](int64_t grp, uint32_t (&wv)[8]) {
        const int64_t w0 = grp * 8;
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
      const int ngroups = (nkb + 1) / 2;
      for (int grp = 0; grp < ngroups && ok; ++grp) {
        load_group(grp + 1, nxt);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int kb = grp * 2 + i;
          if (kb >= nkb) break;
          // Columns c = 0..63 of the stage hold k = 2c, 2c+1; a trailing partial stage
          // (K % 128 != 0) leaves the columns past K at zero.
          const int64_t left = K - (int64_t)kb * kBK;
          const int valid = (int)(left < kBK ? left : kBK) / 2;
          const uint4* bp = reinterpret_cast<const uint4*>(bpair + (int64_t)kb * (kBK / 2)) + 8 * ahalf;
          // Selects keep cur in registers (no runtime index into it).
          const uint32_t wa = i ? (ahalf ? cur[6] : cur[4]) : (ahalf ? cur[2] : cur[0]);
          const uint32_t wb = i ? (ahalf ? cur[7] : cur[5]) : (ahalf ? cur[3] : cur[1]);
          const uint32_t u0 = unzip_bits2(wa), u1 = unzip_bits2(wb);
          uint32_t v[32];
          if (left >= kBK)
            expand_half<false>(u0, u1, bp, 32 * ahalf, valid, v);
          else
            expand_half<true>(u0, u1, bp, 32 * ahalf, valid, v);
          // The previous stage's store has had this stage's arithmetic to land: only now
          // wait for it and release that stage to the MMA.
          flush_pending();
          const int s = (int)(gstage % kStages);
          if (gstage >= kStages) {
            ok = wait_warp(&sh->empty[s], (uint32_t)((gstage / kStages) - 1) & 1u, err, abort_flag, lane);
            if (!ok) break;
            tc_fence_after();
          }
          tmem_st_x32(lane_base + kASlot0 + 64u * s + 32u * ahalf, v);
          pending = s;
          ++gstage;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) cur[i] = nxt[i];
      }
      flush_pending();  // the tile's last stage, before the next tile's sign loads
    }
    flush_pending();
  } else if (warp < kEpiWarp0 + kEpiWarps) {
    // ------------------------------------------------ epilogue: this CTA's 128 rows x kTok tokens
    const int q = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int c0 = 0, c1 = kTok / 32;
    uint16_t* col = reinterpret_cast<uint16_t*>(out_tile) + q * 32 + lane;
    int64_t it = 0;
    for (int64_t tile = pair; tile < tiles; tile += npairs, ++it) {
      if (!wait_warp(&sh->dfull, (uint32_t)it & 1u, err, abort_flag, lane)) break;
      tc_fence_after();
      if (it > 0 && !wait_warp(&sh->stg_free, (uint32_t)(it - 1) & 1u, err, abort_flag, lane)) break;
      const int64_t m0 = (tile / n_blocks) * kTok;
      const int64_t n0 = (tile % n_blocks) * (2 * kRowsCta) + rank * kRowsCta;
      const int64_t nr = n0 + q * 32 + lane;
      const float sc = nr < g.R ? __ldg(g.oscale + nr) : 0.f;
      // The accumulator is read in chunks of 32 columns, two buffers deep: the load of chunk
      // c + 1 is in flight while chunk c is converted and staged, and the accumulator is
      // released to the next tile's MMAs as soon as the last chunk has landed in registers
      // (the MMA waits for that release at every tile boundary).
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(dempty0);
      };
      auto stage_chunk = [&](const uint32_t (&d)[32], int c) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          col[(32 * c + i) * kRowsCta] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(d[i]) * sc));
      };
      static_assert((kTok / 32) % 2 == 0, "chunks are taken in pairs");
      uint32_t da[32], db[32];
      tmem_ld_x32(lane_base + 32u * c0, da);
      tmem_wait_ld_regs(da);
#pragma unroll 1
      for (int c = c0; c < c1; c += 2) {
        // da holds chunk c; chunk c + 1 (< c1: the count is even) goes to db.
        tmem_ld_x32(lane_base + 32u * (c + 1), db);
        stage_chunk(da, c);
        tmem_wait_ld_regs(db);
        if (c + 2 < c1) {
          tmem_ld_x32(lane_base + 32u * (c + 2), da);
          stage_chunk(db, c + 1);
          tmem_wait_ld_regs(da);
        } else {
          release();  // this warp's last read of the accumulator has completed
          stage_chunk(db, c + 1);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->stg_full);
      if (warp == kEpiWarp0 && lane == 0) {
        if (mbar_wait(&sh->stg_full, (uint32_t)it & 1u, err, abort_flag)) {
          tma_store_2d(&tmap_y, out_tile, (int32_t)n0, (int32_t)m0);
          bulk_commit_group();
          bulk_wait_read_all();
        }
        mbar_arrive(&sh->stg_free);
      }
      __syncwarp();
    }
    if (warp == kEpiWarp0 && lane == 0) bulk_wait_all();
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------ TMA producer: this CTA's kTokCta tokens
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      int64_t gstage = 0;
      bool ok = true;
      for (int64_t tile = pair; tile < tiles && ok; tile += npairs) {
        const int32_t y = (int32_t)((tile / n_blocks) * kTok + rank * kTokCta);
        for (int kb = 0; kb < nkb; ++kb, ++gstage) {
          const int s = (int)(gstage % kStages);
          if (gstage >= kStages) {
            ok = mbar_wait_sleep(&sh->empty[s], (uint32_t)((gstage / kStages) - 1) & 1u, err, abort_flag);
            if (!ok) break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&sh->full[s], 2 * kStageBytes);  // both CTAs' bytes
          uint8_t* dst = xs + (size_t)s * kStageBytes;
          tma_load_2d_pair(dst, &tmap_x, full0 + 8u * s, kb * kBK, y);
          tma_load_2d_pair(dst + kSlabBytes, &tmap_x, full0 + 8u * s, kb * kBK + 64, y);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ MMA issuer (rank 0 only)
    if (rank == 0 && lane == 0) {
      const uint32_t xa0 = smem_u32(xs);
      uint64_t d[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) d[j] = sdesc_kmajor_sw128(xa0 + (uint32_t)(j >> 2) * kSlabBytes + 32u * (j & 3));
      uint32_t s = 0, phase = 0;
      int64_t it = 0;
      bool ok = true;
      for (int64_t tile = pair; tile < tiles && ok; tile += npairs, ++it) {
        if (it > 0) {
          ok = mbar_wait(&sh->dempty, (uint32_t)(it - 1) & 1u, err, abort_flag);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kb = 0; kb < nkb; ++kb) {
          ok = mbar_wait(&sh->full[s], phase, err, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t so = (uint64_t)(s * (kStageBytes >> 4));
          const uint32_t aa = tmem + kASlot0 + 64u * s;
          const int64_t rem = K - (int64_t)kb * kBK;
          const int steps = rem >= kBK ? 8 : (int)(rem / 16);  // K % 32 == 0: whole 16-k steps
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < steps) mma_bf16_ts_pair(tmem, aa + 8u * j, d[j] + so, Sh::kIdesc, (kb > 0 || j > 0) ? 1u : 0u);
          mma_commit_pair(&sh->empty[s]);
          if (++s == (uint32_t)kStages) {
            s = 0;
            phase ^= 1u;
          }
        }
        mma_commit_pair(&sh->dfull);
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no MMA, remote arrival or TMA of the pair is still outstanding
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

bool sign_gemm_tc2_supported(const SignGemmArgs& g) {
  return g.K > 0 && g.K <= kMaxK && g.M >= 512 && g.R >= 256 && g.y_dtype == OB_OUT_BF16 && g.ldy % 8 == 0 &&
         (reinterpret_cast<uintptr_t>(g.Y) & 15) == 0;
}

namespace {

template <int kTok>
cudaError_t launch_tc2(const SignGemmArgs& g, const LaunchCtx& c, EncodeTiledFn encode) {
  using Sh = Tc2Shape<kTok>;
  CUtensorMap tmap_x, tmap_y;
  std::memset(&tmap_x, 0, sizeof(tmap_x));
  std::memset(&tmap_y, 0, sizeof(tmap_y));
  {
    const cuuint64_t dims[2] = {(cuuint64_t)g.K, (cuuint64_t)g.M};
    const cuuint64_t strides[1] = {(cuuint64_t)g.K * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)Sh::kTokCta};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(g.X), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)g.R, (cuuint64_t)g.M};
    const cuuint64_t strides[1] = {(cuuint64_t)g.ldy * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kRowsCta, (cuuint32_t)kTok};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.Y, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int64_t tiles = ((g.M + kTok - 1) / kTok) * ((g.R + 2 * kRowsCta - 1) / (2 * kRowsCta));
  const int pairs = (int)std::min<int64_t>(tiles, c.num_sms / 2);
  const size_t smem = 1024 + (size_t)Sh::kStages * Sh::kStageBytes + Sh::kOutTileBytes +
                      sizeof(Tc2Shared<Sh::kStages>) + sizeof(uint32_t) * ((((g.K + 1) / 2) + 3) & ~int64_t(3));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  int na = 1;
  if (c.pdl) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e =
      cudaFuncSetAttribute(sign_gemm_tc2_kernel<kTok>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&cfg, sign_gemm_tc2_kernel<kTok>, tmap_x, tmap_y, g, c.err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool sign_gemm_tc2_narrow(const SignGemmArgs& g, int num_sms) {
  const int64_t wide = ((g.M + 255) / 256) * ((g.R + 2 * kRowsCta - 1) / (2 * kRowsCta));
  return 2 * wide <= num_sms / 2;
}

cudaError_t launch_sign_gemm_tc2(const SignGemmArgs& g, const LaunchCtx& c) {
  if (g.M == 0 || g.R == 0 || g.K == 0) return cudaSuccess;
  if (!sign_gemm_tc2_supported(g)) return cudaErrorInvalidValue;
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(tensor_map_encode_tiled_fn());
  if (!encode) return cudaErrorNotSupported;
  // 128-token tiles when twice as many tiles as the 256-token tiling has still fit one
  // wave of SM pairs (the wide tiling would leave more than half of the pairs idle).
  return sign_gemm_tc2_narrow(g, c.num_sms) ? launch_tc2<128>(g, c, encode) : launch_tc2<256>(g, c, encode);
}

}  // namespace ob
