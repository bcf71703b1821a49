// linear_tc_decode.cu -- small-M sign product on the fifth-generation tensor core.
//
//   Y[m, n] = oscale[n] * sum_k (x[m, k] * iscale[k]) * s[n, k],   M <= 16 per pass
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T;
// for DBF ("Addition is almost all you need ...", "Methodologie") each of the two
// sign products is one call of this kernel.
//
// Design (B200, sm_100a):
//  * The sign matrix is the MMA's A operand and lives in TENSOR MEMORY.  Each of
//    128 threads owns one weight row (one TMEM lane) and expands its packed words
//    straight into bf16 +/-1 pairs with tcgen05.st, so the expanded signs never
//    touch shared memory.  A 32-bit TMEM column holds two bf16 values; the kernel
//    pairs column i with column i+16 of the same packed word, so one shift and
//    one LOP3 produce a column: ((w << (15-i)) & 0x80008000) | 0x3F803F80.
//  * The activations x' = x ⊙ iscale are the B operand (N = 16 tokens, padded
//    with zeros) in shared memory, K-major with the 128-byte swizzle, stored in
//    the same (i, i+16) pairing order so the MMA contracts matching k.
//  * One elected thread issues tcgen05.mma (M=128, N=16, K=16, fp32 accumulate
//    in TMEM) per 16 k; A stages cycle through a ring of TMEM slots guarded by
//    mbarriers (threads -> full, tcgen05.commit -> empty).  An N=16 MMA is
//    short, so a chain of MMAs into one accumulator runs at the MMA latency,
//    not its throughput: k sub-step q of every stage goes to its own
//    accumulator D_q, four independent chains summed in the epilogue.
//  * K is split over the CTAs of a thread-block cluster; the partial 128 x 16
//    tiles are reduced through distributed shared memory, scaled by oscale and
//    stored (bf16 or fp32).  No global workspace and no atomics.
//  * The kernel is latency-bound at decode sizes, so every global load is
//    issued as early as it can be: all of a CTA's packed words go to registers
//    at kernel start, and the first ring of sign stages is expanded into TMEM,
//    before the programmatic-dependent-launch wait -- only the activations
//    depend on the previous kernel in the stream.  The activation loads are
//    all issued before any of them is used.  Weight loads are issued before
//    the TMEM allocation.  Each CTA allocates 256 of the SM's 512 TMEM columns,
//    so two CTAs (of this call or the next) always fit side by side and no
//    allocation can wait on a CTA of its own cluster.
#include <algorithm>
#include <cstdlib>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kRows = 128;          // weight rows per CTA (MMA M)
constexpr int kTok = 16;            // tokens per pass (MMA N)
constexpr int kStageK = 64;         // k per stage (one 128-byte swizzle row of bf16)
constexpr int kAcc = 4;             // independent accumulators: D_q at columns 16q, q < 4
constexpr int kRingBase = 16 * kAcc;
constexpr int kRing = 6;            // TMEM A-slots: columns kRingBase + 32*s, s < 6
constexpr int kTmemCols = 256;      // two CTAs per SM always fit
constexpr int kMaxStagesPerCta = 32;
constexpr int kMaxWords = 2 * kMaxStagesPerCta;
constexpr int kThreads = 160;       // warps 0-3: rows (expand, X' staging, epilogue); warp 4: TMEM + MMA
constexpr uint32_t kAtomBytes = kTok * 128;  // one stage of X': 16 rows x 128 B
constexpr uint32_t kIdesc = idesc_bf16_f32(kRows, kTok);

struct __align__(8) DecodeShared {
  uint64_t full[kRing];
  uint64_t empty[kRing];
  uint64_t dfull;
  uint64_t xready;
  uint32_t tmem_base;
  int abort_flag;
  float part[kTok][kRows];  // partial tile for the cluster reduction
};

__device__ __forceinline__ float ld_dsmem_f32(const float* local_ptr, uint32_t rank) {
  const uint32_t remote = mapa_shared(local_ptr, rank);
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// Expand 32 columns (two packed words, 64 k) of +/-1 bf16 pairs: column c of
// word g holds (k = 32g + c, k = 32g + c + 16) in its (low, high) halves.
__device__ __forceinline__ void expand_stage(uint32_t w0, uint32_t w1, uint32_t (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    v[c] = ((w0 << (15 - c)) & 0x80008000u) | 0x3F803F80u;
    v[16 + c] = ((w1 << (15 - c)) & 0x80008000u) | 0x3F803F80u;
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned* err, volatile int* abort_flag,
                                          int lane) {
  int okw = 1;
  if (lane == 0) okw = mbar_wait(bar, parity, err, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, okw, 0) != 0;
}

template <bool kCluster>
__global__ void __launch_bounds__(kThreads, 2) sign_gemm_tc_decode_kernel(SignGemmArgs g, int64_t m0,
                                                                           int stages_total, int ksplit,
                                                                           unsigned* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // X' atoms first (1024-byte aligned for the swizzle), then the control block.
  uint8_t* xs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int ks = kCluster ? (int)cluster_ctarank() : 0;
  const int st0 = (int)((int64_t)stages_total * ks / ksplit);
  const int st1 = (int)((int64_t)stages_total * (ks + 1) / ksplit);
  const int nst = st1 - st0;
  DecodeShared* sh = reinterpret_cast<DecodeShared*>(xs + (size_t)kMaxStagesPerCta * kAtomBytes);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t K = g.K;
  const int64_t Wd = K / 32;
  const int64_t n0 = (int64_t)blockIdx.y * kRows;
  const int64_t mt = min64(kTok, g.M - m0);

  // Before the previous grid has finished: only L2 prefetches of this CTA's rows.
  if (g.l2_prefetch && warp == 0 && n0 < g.R) {
    const int64_t rows = min64(kRows, g.R - n0);
    const int64_t w_lo = (int64_t)st0 * 2, w_hi = min64(Wd, (int64_t)st1 * 2);
    if ((Wd & 3) == 0 && (w_lo & 3) == 0) {  // 16-byte aligned row pieces
      for (int64_t r = 0; r < rows; ++r)
        if ((r & 31) == lane) prefetch_l2_bulk(g.S + (n0 + r) * Wd + w_lo, (uint32_t)((w_hi - w_lo) * 4));
    }
  }
  pdl_wait();  // every input may have been written by the previous grid in the stream
  pdl_launch_dependents();  // the next grid may start (one grid ahead at most)

  const int64_t n = n0 + (tid & 127);
  const bool row_ok = warp < 4 && n < g.R;
  const int64_t w_begin = (int64_t)st0 * 2;  // even
  const int nw = (int)(min64(Wd, (int64_t)st1 * 2) - w_begin);
  // All of this row's words for the CTA's k range, requested at once.
  uint32_t w[kMaxWords];
  if ((Wd & 1) == 0) {  // rows and w_begin are 8-byte aligned: two words per load
    const uint2* src = reinterpret_cast<const uint2*>(g.S + (row_ok ? n : 0) * Wd + w_begin);
#pragma unroll
    for (int i = 0; i < kMaxWords / 2; ++i) {
      uint2 v = make_uint2(0u, 0u);
      if (row_ok && 2 * i < nw) v = __ldg(src + i);
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
  } else {
    const uint32_t* src = g.S + (row_ok ? n : 0) * Wd + w_begin;
#pragma unroll
    for (int i = 0; i < kMaxWords; ++i) w[i] = (row_ok && i < nw) ? __ldg(src + i) : 0u;
  }
  const float osc = row_ok ? __ldg(g.oscale + n) : 0.f;

  if (tid == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&sh->full[s], 4);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->dfull, 1);
    mbar_init(&sh->xready, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort_flag = &sh->abort_flag;

  if (warp < 4) {
    // ------------------------------------------------ row threads
    const int t = tid;                      // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);


    // First ring round: every slot is free.
#pragma unroll
    for (int j = 0; j < kRing; ++j) {
      if (j < nst) {
        uint32_t v[32];
        expand_stage(w[2 * j], w[2 * j + 1], v);
        tmem_st_x32(lane_base + kRingBase + 32u * j, v);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < kRing; ++j)
        if (j < nst) mbar_arrive(&sh->full[j]);
    }

    // X' = x ⊙ iscale into the swizzled B tile, in (i, i+16) pair order.
    // Unit = (token half h, stage j, word g, 8-column block cb): 8 tokens x 8 pairs.
    {
      const int units = 2 * nst * 4;
      for (int u = t; u < units; u += 128) {
        const int h = u & 1;
        const int rest = u >> 1;
        const int j = rest >> 2;
        const int gw = (rest >> 1) & 1;
        const int cb = rest & 1;
        const int64_t k_lo = (int64_t)(st0 + j) * kStageK + gw * 32 + cb * 8;  // 8 consecutive k
        const int64_t k_hi = k_lo + 16;
        const bool blk_ok = k_lo < K;  // K % 32 == 0: the whole (k_lo, k_hi) block is in or out
        float slo[8], shi[8];
        if (g.iscale && blk_ok) {
          const float4* s4 = reinterpret_cast<const float4*>(g.iscale + k_lo);
          const float4 a0 = __ldg(s4), a1 = __ldg(s4 + 1), b0 = __ldg(s4 + 4), b1 = __ldg(s4 + 5);
          slo[0] = a0.x; slo[1] = a0.y; slo[2] = a0.z; slo[3] = a0.w;
          slo[4] = a1.x; slo[5] = a1.y; slo[6] = a1.z; slo[7] = a1.w;
          shi[0] = b0.x; shi[1] = b0.y; shi[2] = b0.z; shi[3] = b0.w;
          shi[4] = b1.x; shi[5] = b1.y; shi[6] = b1.z; shi[7] = b1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) slo[e] = shi[e] = 1.f;
        }
        uint4 xlo[8], xhi[8];
#pragma unroll
        for (int mm = 0; mm < 8; ++mm) {
          const int m = h * 8 + mm;
          xlo[mm] = make_uint4(0, 0, 0, 0);
          xhi[mm] = make_uint4(0, 0, 0, 0);
          if (m < mt && blk_ok) {
            const uint16_t* xrow = g.X + (m0 + m) * K;
            xlo[mm] = __ldg(reinterpret_cast<const uint4*>(xrow + k_lo));
            xhi[mm] = __ldg(reinterpret_cast<const uint4*>(xrow + k_hi));
          }
        }
        uint8_t* atom = xs + (size_t)j * kAtomBytes;
        const uint32_t e0 = (uint32_t)(gw * 32 + cb * 16);  // element index of pair (gw*16 + cb*8)
#pragma unroll
        for (int mm = 0; mm < 8; ++mm) {
          const int m = h * 8 + mm;
          const uint32_t lo_w[4] = {xlo[mm].x, xlo[mm].y, xlo[mm].z, xlo[mm].w};
          const uint32_t hi_w[4] = {xhi[mm].x, xhi[mm].y, xhi[mm].z, xhi[mm].w};
          uint32_t out[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t lw = lo_w[e >> 1], hw = hi_w[e >> 1];
            const float xl = __uint_as_float((e & 1) ? (lw & 0xFFFF0000u) : (lw << 16)) * slo[e];
            const float xh = __uint_as_float((e & 1) ? (hw & 0xFFFF0000u) : (hw << 16)) * shi[e];
            out[e] = pack_bf16x2(xl, xh);
          }
          *reinterpret_cast<uint4*>(atom + sw128_offset(m, e0)) = make_uint4(out[0], out[1], out[2], out[3]);
          *reinterpret_cast<uint4*>(atom + sw128_offset(m, e0 + 8)) = make_uint4(out[4], out[5], out[6], out[7]);
        }
      }
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (t == 0) mbar_arrive(&sh->xready);
    }

    // Remaining stages through the ring, from the words already in registers.
    bool ok = true;
#pragma unroll
    for (int j = kRing; j < kMaxStagesPerCta; ++j) {
      if (j >= nst || !ok) break;
      const int slot = j % kRing;
      uint32_t v[32];
      expand_stage(w[2 * j], w[2 * j + 1], v);
      ok = warp_wait(&sh->empty[slot], (uint32_t)((j / kRing) - 1) & 1u, err, abort_flag, lane);
      if (!ok) break;
      tc_fence_after();
      tmem_st_x32(lane_base + kRingBase + 32u * slot, v);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->full[slot]);
    }

    // Epilogue: this row's 16 partial sums.
    float acc[kTok];
    ok = warp_wait(&sh->dfull, 0, err, abort_flag, lane) && ok;
    tc_fence_after();
    {
      // D_2 and D_3 hold data only if the CTA's first stage is a full 64-k stage.
      const int nacc = ((int64_t)st0 * kStageK + 32 < K) ? kAcc : 2;
      uint32_t d[kAcc][16];
#pragma unroll
      for (int q = 0; q < kAcc; ++q) tmem_ld_x16(lane_base + 16u * q, d[q]);
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < kTok; ++m) {
        float v = __uint_as_float(d[0][m]) + __uint_as_float(d[1][m]);
        if (nacc == kAcc) v += __uint_as_float(d[2][m]) + __uint_as_float(d[3][m]);
        acc[m] = ok ? v : 0.f;
      }
    }
    if constexpr (!kCluster) {
      if (row_ok) {
#pragma unroll
        for (int m = 0; m < kTok; ++m) {
          if (m >= mt) break;
          const int64_t off = (m0 + m) * g.ldy + n;
          if (g.y_dtype == OB_OUT_F32)
            static_cast<float*>(g.Y)[off] = acc[m] * osc;
          else
            static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(acc[m] * osc);
        }
      }
    } else {
#pragma unroll
      for (int m = 0; m < kTok; ++m) sh->part[m][t] = acc[m];
    }
  } else {
    // ------------------------------------------------ warp 4: MMA issue (one elected lane)
    if (lane == 0) {
      bool ok = mbar_wait(&sh->xready, 0, err, abort_flag);
      for (int j = 0; j < nst && ok; ++j) {
        const int slot = j % kRing;
        ok = mbar_wait(&sh->full[slot], (uint32_t)(j / kRing) & 1u, err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xs_atom = smem_u32(xs) + (uint32_t)j * kAtomBytes;
        const int64_t k_stage = (int64_t)(st0 + j) * kStageK;
        const int ksub = (k_stage + 32 < K) ? 4 : 2;  // last stage may hold one word
        for (int q = 0; q < ksub; ++q) {
          const uint64_t bdesc = sdesc_kmajor_sw128(xs_atom + 32u * q);
          mma_bf16_ts(tmem + 16u * q, tmem + kRingBase + 32u * slot + 8u * q, bdesc, kIdesc, j > 0 ? 1u : 0u);
        }
        mma_commit(&sh->empty[slot]);
      }
      mma_commit(&sh->dfull);  // also covers abort: arrives once prior MMAs retire
    }
    __syncwarp();
  }

  if constexpr (kCluster) {
    // Rank ks reduces rows [ks*128/ksplit, (ks+1)*128/ksplit) over all CTAs of the cluster.
    const int r0 = kRows * ks / ksplit, r1 = kRows * (ks + 1) / ksplit;
    const int rows = r1 - r0;
    const int my_r = r0 + tid % rows;  // each thread keeps one row (kThreads is a multiple of rows or more)
    const float my_osc = (n0 + my_r < g.R) ? __ldg(g.oscale + n0 + my_r) : 0.f;
    cluster_sync_all();
    if (!*abort_flag) {
      for (int idx = tid; idx < rows * (int)mt; idx += kThreads) {
        const int m = idx / rows;
        const int r = r0 + (idx - m * rows);
        const int64_t n = n0 + r;
        if (n >= g.R) continue;
        float parts[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) parts[q] = q < ksplit ? ld_dsmem_f32(&sh->part[m][r], (uint32_t)q) : 0.f;
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) s += parts[q];
        s *= (r == my_r) ? my_osc : __ldg(g.oscale + n);
        const int64_t off = (m0 + m) * g.ldy + n;
        if (g.y_dtype == OB_OUT_F32)
          static_cast<float*>(g.Y)[off] = s;
        else
          static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(s);
      }
    }
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

int env_int(const char* name, int dflt) {
  const char* s = std::getenv(name);
  return s ? std::atoi(s) : dflt;
}

// K-split over the cluster: with two CTAs per SM, minimise the per-SM share of
// the work; prefer fewer splits on ties.
int choose_ksplit(int64_t row_blocks, int stages, int num_sms) {
  const int forced = env_int("OB_DECODE_KSPLIT", 0);
  auto fits = [&](int ks) { return ks <= stages && (stages + ks - 1) / ks <= kMaxStagesPerCta; };
  if (forced > 0 && forced <= 8 && fits(forced)) return forced;
  int best = 0;
  double best_cost = 1e30;
  for (int ks = 1; ks <= 8; ++ks) {
    if (!fits(ks)) continue;
    const int64_t ctas = row_blocks * ks;
    const double cost = (double)((ctas + num_sms - 1) / num_sms) / ks;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = ks;
    }
  }
  return best;
}

}  // namespace

cudaError_t launch_sign_gemm_tc_decode(const SignGemmArgs& g, const LaunchCtx& c) {
  const int stages = (int)((g.K + kStageK - 1) / kStageK);
  const int64_t row_blocks = (g.R + kRows - 1) / kRows;
  if (stages == 0 || row_blocks == 0 || g.M == 0) return cudaSuccess;
  const int ksplit = choose_ksplit(row_blocks, stages, c.num_sms);
  if (ksplit == 0) return cudaErrorInvalidValue;  // K too large for one cluster of this kernel
  const size_t smem = 1024 + (size_t)kMaxStagesPerCta * kAtomBytes + sizeof(DecodeShared);

  for (int64_t m0 = 0; m0 < g.M; m0 += kTok) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ksplit, (unsigned)row_blocks, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (ksplit > 1) {
      attrs[na].id = cudaLaunchAttributeClusterDimension;
      attrs[na].val.clusterDim.x = (unsigned)ksplit;
      attrs[na].val.clusterDim.y = 1;
      attrs[na].val.clusterDim.z = 1;
      ++na;
    }
    if (c.pdl) {
      attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attrs[na].val.programmaticStreamSerializationAllowed = 1;
      ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    cudaError_t e;
    if (ksplit > 1) {
      auto kern = sign_gemm_tc_decode_kernel<true>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, kern, g, m0, stages, ksplit, c.err);
    } else {
      auto kern = sign_gemm_tc_decode_kernel<false>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, kern, g, m0, stages, ksplit, c.err);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace ob
