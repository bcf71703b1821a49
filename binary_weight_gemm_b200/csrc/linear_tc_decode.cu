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
//    mbarriers (threads -> full, tcgen05.commit -> empty).
//  * K is split over the CTAs of a thread-block cluster; the partial 128 x 16
//    tiles are reduced through distributed shared memory, scaled by oscale and
//    stored (bf16 or fp32).  No global workspace and no atomics.
//  * Weight words are requested before the programmatic-dependent-launch wait
//    and the first ring of sign stages is expanded before it too: only the
//    activations depend on the previous kernel in the stream.
#include <algorithm>
#include <cstdlib>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kRows = 128;          // weight rows per CTA (MMA M)
constexpr int kTok = 16;            // tokens per pass (MMA N)
constexpr int kStageK = 64;         // k per stage (one 128-byte swizzle row of bf16)
constexpr int kRing = 6;            // TMEM A-slots
constexpr int kTmemCols = 256;      // D at columns [0,16), A slots at 32 + 32*s
constexpr int kMaxStagesPerCta = 48;
constexpr int kThreads = 160;       // warps 0-3: rows (unpack, X' prep, epilogue); warp 4: TMEM + MMA
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

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(const float* local_ptr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local_ptr)), "r"(rank));
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

template <bool kCluster>
__global__ void __launch_bounds__(kThreads) sign_gemm_tc_decode_kernel(SignGemmArgs g, int64_t m0,
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
  pdl_launch_dependents();

  if (warp < 4) {
    // ------------------------------------------------ row threads
    const int t = tid;                      // row within the tile == TMEM lane
    const int64_t n = n0 + t;
    const bool row_ok = n < g.R;
    const uint32_t* srow = g.S + (row_ok ? n : 0) * Wd;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int64_t w_begin = (int64_t)st0 * 2;
    const int64_t w_end = min64(Wd, (int64_t)st1 * 2);

    // Words of ring round r (stages r*kRing .. r*kRing+kRing-1) of this row.
    auto load_round = [&](uint32_t (&buf)[2 * kRing], int r) {
#pragma unroll
      for (int i = 0; i < 2 * kRing; ++i) {
        const int64_t w = w_begin + (int64_t)r * 2 * kRing + i;
        buf[i] = (row_ok && w < w_end) ? __ldg(srow + w) : 0u;
      }
    };
    // Expand round r into the ring (round 0 finds every slot free).
    auto process_round = [&](const uint32_t (&buf)[2 * kRing], int r) -> bool {
#pragma unroll
      for (int jj = 0; jj < kRing; ++jj) {
        const int j = r * kRing + jj;
        if (j >= nst) break;
        uint32_t v[32];
        expand_stage(buf[2 * jj], buf[2 * jj + 1], v);
        if (r > 0) {
          int okw = 1;
          if (lane == 0) okw = mbar_wait(&sh->empty[jj], (uint32_t)(r - 1) & 1u, err, abort_flag) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, okw, 0)) return false;
          tc_fence_after();
        }
        tmem_st_x32(lane_base + 32u + 32u * jj, v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->full[jj]);
      }
      return true;
    };

    // Weight words do not depend on the previous grid: request two rounds and
    // expand the first before the dependency wait.
    uint32_t wa[2 * kRing], wb[2 * kRing];
    load_round(wa, 0);
    load_round(wb, 1);
    bool ok = process_round(wa, 0);

    // Activations depend on the previous grid in the stream.
    pdl_wait();

    // X' = x ⊙ iscale into the swizzled B tile, in (i, i+16) pair order.
    // Unit = (token half h, stage j, word g, 8-column block cb): 8 pairs -> 32 bytes.
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
        float slo[8], shi[8];
        const bool lo_ok = k_lo < K, hi_ok = k_hi < K;  // K % 32 == 0: blocks are all-in or all-out
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          slo[e] = (g.iscale && lo_ok) ? __ldg(g.iscale + k_lo + e) : 1.f;
          shi[e] = (g.iscale && hi_ok) ? __ldg(g.iscale + k_hi + e) : 1.f;
        }
        uint8_t* atom = xs + (size_t)j * kAtomBytes;
#pragma unroll 2
        for (int mm = 0; mm < 8; ++mm) {
          const int m = h * 8 + mm;
          uint4 xlo = make_uint4(0, 0, 0, 0), xhi = make_uint4(0, 0, 0, 0);
          if (m < mt) {
            const uint16_t* xrow = g.X + (m0 + m) * K;
            if (lo_ok) xlo = __ldg(reinterpret_cast<const uint4*>(xrow + k_lo));
            if (hi_ok) xhi = __ldg(reinterpret_cast<const uint4*>(xrow + k_hi));
          }
          const uint32_t lo_w[4] = {xlo.x, xlo.y, xlo.z, xlo.w};
          const uint32_t hi_w[4] = {xhi.x, xhi.y, xhi.z, xhi.w};
          uint32_t out[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t lw = lo_w[e >> 1], hw = hi_w[e >> 1];
            const float xl = __uint_as_float((e & 1) ? (lw & 0xFFFF0000u) : (lw << 16)) * slo[e];
            const float xh = __uint_as_float((e & 1) ? (hw & 0xFFFF0000u) : (hw << 16)) * shi[e];
            out[e] = pack_bf16x2(xl, xh);
          }
          // Pair index within the stage row: gw*16 + cb*8 + e -> element 2*(that).
          const uint32_t e0 = (uint32_t)(gw * 32 + cb * 16);
          *reinterpret_cast<uint4*>(atom + sw128_offset(m, e0)) = make_uint4(out[0], out[1], out[2], out[3]);
          *reinterpret_cast<uint4*>(atom + sw128_offset(m, e0 + 8)) = make_uint4(out[4], out[5], out[6], out[7]);
        }
      }
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (t == 0) mbar_arrive(&sh->xready);
    }

    // Remaining rounds, loads one round ahead (two register buffers, unrolled by two).
    for (int r = 1; ok && r * kRing < nst; r += 2) {
      load_round(wa, r + 1);
      ok = process_round(wb, r);
      if (!ok || (r + 1) * kRing >= nst) break;
      load_round(wb, r + 2);
      ok = process_round(wa, r + 1);
    }

    // Epilogue: this row's 16 partial sums.
    float acc[kTok];
    {
      int okw = 1;
      if (lane == 0) okw = mbar_wait(&sh->dfull, 0, err, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, okw, 0) && ok;
    }
    tc_fence_after();
    {
      uint32_t d[16];
      tmem_ld_x16(lane_base, d);
      tmem_wait_ld();
#pragma unroll
      for (int m = 0; m < kTok; ++m) acc[m] = ok ? __uint_as_float(d[m]) : 0.f;
    }
    if constexpr (!kCluster) {
      if (row_ok) {
        const float sc = __ldg(g.oscale + n);
#pragma unroll
        for (int m = 0; m < kTok; ++m) {
          if (m >= mt) break;
          const int64_t off = (m0 + m) * g.ldy + n;
          if (g.y_dtype == OB_OUT_F32)
            static_cast<float*>(g.Y)[off] = acc[m] * sc;
          else
            static_cast<__nv_bfloat16*>(g.Y)[off] = __float2bfloat16_rn(acc[m] * sc);
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
          mma_bf16_ts(tmem, tmem + 32u + 32u * slot + 8u * q, bdesc, kIdesc, (j > 0 || q > 0) ? 1u : 0u);
        }
        mma_commit(&sh->empty[slot]);
      }
      mma_commit(&sh->dfull);  // also covers abort: arrives once prior MMAs retire
    }
    __syncwarp();
    pdl_wait();  // this warp stores Y in the cluster reduction below
  }

  if constexpr (kCluster) {
    cluster_sync_all();
    // Rank ks reduces rows [ks*128/ksplit, (ks+1)*128/ksplit) over all CTAs of the cluster.
    const int r0 = kRows * ks / ksplit, r1 = kRows * (ks + 1) / ksplit;
    const int rows = r1 - r0;
    if (!*abort_flag) {
      for (int idx = tid; idx < rows * (int)mt; idx += kThreads) {
        const int m = idx / rows;
        const int r = r0 + (idx - m * rows);
        const int64_t n = n0 + r;
        if (n >= g.R) continue;
        float s = 0.f;
        for (int q = 0; q < ksplit; ++q) s += ld_dsmem_f32(&sh->part[m][r], (uint32_t)q);
        s *= __ldg(g.oscale + n);
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

// K-split over the cluster: minimise the per-SM share of the work, prefer fewer splits.
int choose_ksplit(int64_t row_blocks, int stages, int num_sms) {
  const int forced = env_int("OB_DECODE_KSPLIT", 0);
  int best = 1;
  double best_cost = 1e30;
  for (int ks = 1; ks <= 8; ++ks) {
    if (ks > stages) break;
    if ((stages + ks - 1) / ks > kMaxStagesPerCta) continue;
    const int64_t ctas = row_blocks * ks;
    const double cost = (double)((ctas + num_sms - 1) / num_sms) / ks;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = ks;
    }
  }
  if (forced > 0 && forced <= 8 && forced <= stages && (stages + forced - 1) / forced <= kMaxStagesPerCta)
    best = forced;
  return best;
}

}  // namespace

cudaError_t launch_sign_gemm_tc_decode(const SignGemmArgs& g, const LaunchCtx& c) {
  const int stages = (int)((g.K + kStageK - 1) / kStageK);
  const int64_t row_blocks = (g.R + kRows - 1) / kRows;
  if (stages == 0 || row_blocks == 0 || g.M == 0) return cudaSuccess;
  if ((stages + 7) / 8 > kMaxStagesPerCta) return cudaErrorInvalidValue;  // K too large for this kernel
  const int ksplit = choose_ksplit(row_blocks, stages, c.num_sms);
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
