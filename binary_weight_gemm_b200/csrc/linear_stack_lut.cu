// linear_stack_lut.cu -- a list of one-token sign-product layers in one persistent
// launch, by table lookup, with every CTA's sign rows staged in shared memory.
//
//   y[n] = oscale[n] * sum_k (x[k] * iscale[k]) * s[n, k]
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": y = [(x ⊙ b^T) W_sign^T] ⊙ a^T,
// applied layer after layer as in a decoder (the barrier groups of stack_common.cuh).
//
// At one token every sign is used once, so the work is a stream of weight bits
// through the SMs.  What limits the warp-MMA stack at one token is the chain of
// latencies of each 32-row block (activations from L2, signs from L2, MMA), and
// the MMA itself wastes 7 of its 8 token columns.  Here:
//  * The rows of a barrier group (its layers concatenated) are split into one
//    contiguous range per CTA.  A CTA's range is at most a few segments (one per
//    layer it touches), each a contiguous run of packed sign rows, which one bulk
//    copy (the copy engine, completion on an mbarrier) brings into shared memory.
//    Weights do not depend on activations, so the copies for group g+1 are issued
//    when group g starts (two staging buffers): the signs are on chip by the time
//    the grid barrier releases the CTA.
//  * Per 1024 k (a "chunk") the CTA tabulates, for every 4 consecutive k, the 16
//    signed sums ±x'_0 ±x'_1 ±x'_2 ±x'_3 (x' = x ⊙ b) in shared memory; a packed
//    nibble then costs one shift/mask, one table load and one add.  Entry v of
//    (word q, nibble j) sits at float v*256 + j*32 + q, so lane q, which reads word
//    q of the chunk, always reads bank q.  Tables are double-buffered: one CTA
//    barrier per chunk.  The activations of the chunk after next are loaded (through
//    L2: other CTAs of this grid wrote them) while the current chunk is consumed; the
//    scale vectors of the next group are prefetched into L2 with its sign rows.
//  * Warp w holds the partial sums of rows w, w+16, ... (12 per warp, 192 rows per
//    pass of a segment) in registers across the chunks.
// The launcher uses this form only when asked (OB_STACK_LUT=1) and every CTA's share
// of every group fits one staging buffer (stack_lut_fits); otherwise the MMA form runs.
// Measured on B200 for one token through 32 blocks of 7B-shaped layers: 2118 us per
// token against 1769 us for the MMA form.  DRAM traffic equals the packed weights (no
// re-reads); the largest stall is the CTA barrier (one per 1024-k chunk, load imbalance
// between warps when a CTA holds few rows, and the grid barrier).
#include <algorithm>

#include <cuda_bf16.h>

#include "stack_common.cuh"

namespace ob {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerWarp = 12;
constexpr int kPassRows = kWarps * kRowsPerWarp;  // 192
constexpr int kChunkWords = 32;                   // 1024 k per table
constexpr int kTableFloats = 16 * 8 * kChunkWords;  // 16 KB
constexpr uint32_t kSignBuf = 80u * 1024u;          // one group's sign rows of one CTA
constexpr int kMaxSeg = 48;
constexpr uint32_t kTableBytes = sizeof(float) * kTableFloats;  // 16 KB: tables sit on 16 KB boundaries
// Up to 16 KB of alignment slack, two tables, two staging buffers.
constexpr size_t kDynSmem = kTableBytes + 2 * (size_t)kTableBytes + 2 * (size_t)kSignBuf;

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
template <int kOff>
__device__ __forceinline__ float lds_f32_off(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(kOff));
  return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Sum of the 8 table entries that the packed word w selects, one per nibble.  tl is the
// shared address of this lane's column of the table (16 KB aligned base + 4 * lane), so
// (value << 10) can be OR'ed in; nibble j's block of the table is j * 128 bytes on.
__device__ __forceinline__ float word_sum(uint32_t w, uint32_t tl) {
  float a = lds_f32(((w << 10) & 0x3C00u) | tl);
  float b = lds_f32_off<128>(((w << 6) & 0x3C00u) | tl);
  a += lds_f32_off<256>(((w << 2) & 0x3C00u) | tl);
  b += lds_f32_off<384>(((w >> 2) & 0x3C00u) | tl);
  a += lds_f32_off<512>(((w >> 6) & 0x3C00u) | tl);
  b += lds_f32_off<640>(((w >> 10) & 0x3C00u) | tl);
  a += lds_f32_off<768>(((w >> 14) & 0x3C00u) | tl);
  b += lds_f32_off<896>(((w >> 18) & 0x3C00u) | tl);
  return a + b;
}

struct Seg {
  int64_t n0;     // first row within the layer
  int32_t layer;  // index into the list
  int32_t rows;
  uint32_t soff;  // byte offset of the rows in the staging buffer
};

struct SegList {
  int n;
  Seg s[kMaxSeg];
};

// CTA c's share [lo, hi) of a group of R rows on G CTAs (the same on host and device).
__host__ __device__ __forceinline__ void cta_range(int64_t R, int c, int G, int64_t* lo, int64_t* hi) {
  *lo = R * c / G;
  *hi = R * (c + 1) / G;
}

// Contiguous global -> shared copy by the bulk-copy engine, completion counted in bytes
// on `bar` (this CTA's).  dst and src 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_load_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// One thread: the segments of CTA c in the group [l, e) into `out`, and the bulk copies
// of their sign rows into `buf`, completing on `bar`.  Whether they fit was checked on
// the host; a list that does not fit is cut short (and its rows left unwritten) rather
// than overrun the buffer, with the error recorded.
__device__ void issue_group(const StackParams& p, int l, int e, int c, int G, SegList& out, uint8_t* buf,
                            uint64_t* bar) {
  int64_t R = 0;
  for (int li = l; li < e; ++li) R += p.L[li].N;
  int64_t lo, hi;
  cta_range(R, c, G, &lo, &hi);
  int64_t base = 0;
  uint32_t soff = 0;
  int n = 0;
  for (int li = l; li < e && base < hi; ++li) {
    const StackLayer& L = p.L[li];
    const int64_t s = lo > base ? lo : base, t = hi < base + L.N ? hi : base + L.N;
    if (s < t) {
      const uint64_t bytes = (uint64_t)(t - s) * (uint64_t)(L.K / 8);
      if (n == kMaxSeg || soff + bytes > kSignBuf) {
        record_error(p.err, OB_DEVERR_BOUNDS);
        break;
      }
      out.s[n] = Seg{s - base, li, (int32_t)(t - s), soff};
      ++n;
      soff += (uint32_t)bytes;
    }
    base += L.N;
  }
  out.n = n;
  mbar_arrive_expect_tx(bar, soff);
  for (int i = 0; i < n; ++i) {
    const Seg& sg = out.s[i];
    const StackLayer& L = p.L[sg.layer];
    bulk_load_g2s(buf + sg.soff, L.S + sg.n0 * (L.K / 32), (uint32_t)sg.rows * (uint32_t)(L.K / 8), bar);
  }
  // The scale vectors are read with plain loads, one chunk at a time: bring them into L2
  // now (a hint) so that those loads do not wait on HBM.  The output-scale range is cut
  // to whole 16-byte pieces inside the array.
  for (int i = 0; i < n; ++i) {
    const Seg& sg = out.s[i];
    const StackLayer& L = p.L[sg.layer];
    if (L.iscale) prefetch_l2_bulk(L.iscale, (uint32_t)(L.K * 4));
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(L.oscale + sg.n0);
    const uintptr_t o1 = reinterpret_cast<uintptr_t>(L.oscale + sg.n0 + sg.rows);
    const uintptr_t a0 = o0 & ~(uintptr_t)15;
    if (o1 > a0) prefetch_l2_bulk(reinterpret_cast<const void*>(a0), (uint32_t)(o1 - a0));
  }
}

// This thread's 4 activations and input scales of chunk `ch` of layer L (zeros past K).
// Thread t tabulates word q = t % 32, nibble j = (t / 32) % 8, values 8h .. 8h+7 (h = t / 256).
__device__ __forceinline__ void load_x(const StackLayer& L, int ch, uint2& xv, float4& sc) {
  const int q = threadIdx.x & 31, j = (threadIdx.x >> 5) & 7;
  const int64_t word = (int64_t)ch * kChunkWords + q;
  xv = make_uint2(0u, 0u);
  sc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (word < L.K / 32) {
    const int64_t k = word * 32 + 4 * j;
    xv = __ldcg(reinterpret_cast<const uint2*>(L.X + k));
    sc = L.iscale ? __ldg(reinterpret_cast<const float4*>(L.iscale + k)) : make_float4(1.f, 1.f, 1.f, 1.f);
  }
}

// Write this thread's 8 table entries.  Bit b of the value v set <=> the sign of x'_b is -1.
__device__ __forceinline__ void build_table(float* tab, uint2 xv, float4 sc) {
  const int q = threadIdx.x & 31, j = (threadIdx.x >> 5) & 7, h = threadIdx.x >> 8;
  const float x0 = __uint_as_float(xv.x << 16) * sc.x;
  const float x1 = __uint_as_float(xv.x & 0xFFFF0000u) * sc.y;
  const float x2 = __uint_as_float(xv.y << 16) * sc.z;
  const float x3 = __uint_as_float(xv.y & 0xFFFF0000u) * sc.w;
  const float p[4] = {x0 + x1, -x0 + x1, x0 - x1, -x0 - x1};
  // Values v = 8h + u, u < 8: bits 0, 1 of v are u & 3, bit 2 is u >> 2, bit 3 is h.
  const float x3s = h ? -x3 : x3;
  const float hh[2] = {x2 + x3s, -x2 + x3s};
  float* dst = tab + (8 * h) * 256 + j * 32 + q;
#pragma unroll
  for (int u = 0; u < 8; ++u) dst[u * 256] = p[u & 3] + hh[u >> 2];
}

// Position in a CTA's items of one group: segment s, pass, chunk ch.  Past the end: s == n.
struct Cursor {
  int s, pass, ch;
};

__device__ __forceinline__ Cursor advance(const StackParams& p, const SegList& sl, Cursor c) {
  if (c.s >= sl.n) return c;
  const Seg& sg = sl.s[c.s];
  const int64_t Wd = p.L[sg.layer].K / 32;
  const int nch = (int)((Wd + kChunkWords - 1) / kChunkWords);
  const int passes = (sg.rows + kPassRows - 1) / kPassRows;
  if (++c.ch == nch) {
    c.ch = 0;
    if (++c.pass == passes) {
      c.pass = 0;
      ++c.s;
    }
  }
  return c;
}

__global__ void __launch_bounds__(kThreads, 1) sign_stack_lut_kernel(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ SegList lists[2];
  __shared__ __align__(8) uint64_t mbar[2];
  __shared__ int s_ok;
  __shared__ int s_abort;
  // [slack to a 16 KB boundary][table 0][table 1][staging 0][staging 1]
  const uint32_t dsm_s = smem_u32(dsm);
  const uint32_t tab_off = ((dsm_s + kTableBytes - 1) & ~(kTableBytes - 1)) - dsm_s;
  float* const tab0 = reinterpret_cast<float*>(dsm + tab_off);
  uint8_t* const sbuf = dsm + tab_off + 2 * kTableBytes;
  const int G = gridDim.x, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    fence_mbar_init();
    s_abort = 0;
  }
  pdl_wait();  // the first layers' inputs may come from the previous grid in the stream
  int e = group_end(p, 0);
  if (threadIdx.x == 0) issue_group(p, 0, e, c, G, lists[0], sbuf, &mbar[0]);
  __syncthreads();

  unsigned barriers = 0;
  uint32_t tc = 0;  // chunks consumed so far: selects the table buffer
  int gi = 0;
  for (int l = 0; l < p.n; ++gi) {
    const int b = gi & 1;
    const int e2 = e < p.n ? group_end(p, e) : e;
    // The other buffer was last read in group gi - 1, which every thread of this CTA
    // finished before the grid barrier; order those reads before the async writes.
    if (threadIdx.x == 0 && e < p.n) {
      fence_proxy_async_smem();
      issue_group(p, e, e2, c, G, lists[b ^ 1], sbuf + (size_t)(b ^ 1) * kSignBuf, &mbar[b ^ 1]);
    }
    const bool staged = mbar_wait(&mbar[b], (uint32_t)(gi >> 1) & 1u, p.err, &s_abort);
    // One verdict for the whole CTA: a thread that gave up just before the copies
    // landed must not leave the others waiting at a CTA barrier.
    if (__syncthreads_or(!staged)) {
      // Leave the grid; let the other CTAs leave at their next barrier.  The copies of
      // the next group are waited for (bounded) before the shared memory goes away.
      if (threadIdx.x == 0) {
        atomicExch(p.bar + 1, 1u);
        if (e < p.n) mbar_wait_limit(&mbar[b ^ 1], (uint32_t)((gi + 1) >> 1) & 1u, p.err, nullptr, 100000000ull);
      }
      return;
    }
    const SegList& sl = lists[b];
    const uint8_t* gbuf = sbuf + (size_t)b * kSignBuf;
    if (sl.n > 0) {
      // Items are (segment, pass, chunk) in order.  The activations of item t + 2 are
      // loaded while item t is consumed: two chunks of cover for the L2 round trip.
      Cursor cur{0, 0, 0}, n1 = advance(p, sl, cur), n2 = advance(p, sl, n1);
      uint2 xa, xb = make_uint2(0u, 0u);
      float4 sa, sb = make_float4(0.f, 0.f, 0.f, 0.f);
      load_x(p.L[sl.s[0].layer], 0, xa, sa);
      if (n1.s < sl.n) load_x(p.L[sl.s[n1.s].layer], n1.ch, xb, sb);
      float acc[kRowsPerWarp], osc[kRowsPerWarp];
      for (;;) {
        const Seg sg = sl.s[cur.s];
        const StackLayer& L = p.L[sg.layer];
        const int64_t Wd = L.K / 32;
        const int nch = (int)((Wd + kChunkWords - 1) / kChunkWords);
        float* tab = tab0 + (tc & 1u) * kTableFloats;
        build_table(tab, xa, sa);
        xa = xb;
        sa = sb;
        if (n2.s < sl.n) load_x(p.L[sl.s[n2.s].layer], n2.ch, xb, sb);
        if (cur.ch == 0) {
#pragma unroll
          for (int i = 0; i < kRowsPerWarp; ++i) {
            const int r = cur.pass * kPassRows + warp + kWarps * i;
            acc[i] = 0.f;
            osc[i] = (lane == 0 && r < sg.rows) ? __ldg(L.oscale + sg.n0 + r) : 0.f;
          }
        }
        __syncthreads();  // the table is complete; the buffer written next was last read two chunks ago

        // Rows pass * 192 + warp + 16 i, i < nr, of this segment; word wi of each.
        const int wi = cur.ch * kChunkWords + lane;
        const bool wvalid = wi < Wd;
        const int rows_left = sg.rows - cur.pass * kPassRows - warp;
        const int nr = rows_left <= 0 ? 0 : min(kRowsPerWarp, (rows_left + kWarps - 1) / kWarps);
        const uint32_t rstride = (uint32_t)(kWarps * Wd * 4);
        const uint32_t a0 = smem_u32(gbuf) + sg.soff + (uint32_t)(((cur.pass * kPassRows + warp) * Wd + wi) * 4);
        const uint32_t tl = smem_u32(tab) + (uint32_t)lane * 4u;
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; i += 2) {
          if (i < nr) {  // warp-uniform; row i + 1 may be past the end: its word reads as 0 and its sum is unused
            const uint32_t w0 = wvalid ? lds_u32(a0 + (uint32_t)i * rstride) : 0u;
            const uint32_t w1 = (wvalid && i + 1 < nr) ? lds_u32(a0 + (uint32_t)(i + 1) * rstride) : 0u;
            acc[i] += word_sum(w0, tl);
            acc[i + 1] += word_sum(w1, tl);
          }
        }
        if (cur.ch == nch - 1) {
#pragma unroll
          for (int i = 0; i < kRowsPerWarp; ++i) {
            const int r = cur.pass * kPassRows + warp + kWarps * i;
            if (r < sg.rows) {
              float v = acc[i];
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              if (lane == 0) {
                const int64_t n = sg.n0 + r;
                v *= osc[i];
                if (L.y_dtype == OB_OUT_F32)
                  static_cast<float*>(L.Y)[n] = v;
                else
                  static_cast<__nv_bfloat16*>(L.Y)[n] = __float2bfloat16_rn(v);
              }
            }
          }
        }
        ++tc;
        if (n1.s >= sl.n) break;
        cur = n1;
        n1 = n2;
        n2 = advance(p, sl, n2);
      }
    }
    l = e;
    e = e2;
    if (l < p.n) {
      ++barriers;
      if (!grid_barrier(p.bar, barriers * (unsigned)G, p.err, &s_ok)) {
        if (threadIdx.x == 0)
          mbar_wait_limit(&mbar[b ^ 1], (uint32_t)((gi + 1) >> 1) & 1u, p.err, nullptr, 100000000ull);
        return;
      }
    }
  }
}

}  // namespace

bool stack_lut_fits(const StackParams& p, int G) {
  if (p.M != 1 || G < 1) return false;
  for (int i = 0; i < p.n; ++i)
    if (p.L[i].K % 128 != 0 || (reinterpret_cast<uintptr_t>(p.L[i].S) & 15) != 0) return false;
  for (int l = 0; l < p.n;) {
    int e = l + 1;
    while (e < p.n && !p.L[e].barrier) ++e;
    int64_t R = 0, maxrow = 0;
    for (int li = l; li < e; ++li) {
      R += p.L[li].N;
      maxrow = std::max<int64_t>(maxrow, p.L[li].K / 8);
    }
    // A CTA holds at most ceil(R / G) rows: enough when those fit at the widest row.
    const int64_t share = (R + G - 1) / G;
    if (!(e - l <= kMaxSeg && share * maxrow <= (int64_t)kSignBuf)) {
      for (int c = 0; c < G; ++c) {
        int64_t lo, hi;
        cta_range(R, c, G, &lo, &hi);
        int64_t base = 0, bytes = 0;
        int n = 0;
        for (int li = l; li < e; ++li) {
          const int64_t s = std::max(lo, base), t = std::min(hi, base + p.L[li].N);
          if (s < t) {
            ++n;
            bytes += (t - s) * (p.L[li].K / 8);
          }
          base += p.L[li].N;
        }
        if (n > kMaxSeg || bytes > (int64_t)kSignBuf) return false;
      }
    }
    l = e;
  }
  return true;
}

cudaError_t launch_stack_lut(const StackParams& prm, const LaunchCtx& c) {
  cudaError_t e = cudaFuncSetAttribute(sign_stack_lut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kDynSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sign_stack_lut_kernel, kThreads, kDynSmem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)c.num_sms, 1, 1);  // one CTA per SM: all resident (cooperative)
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kDynSmem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, sign_stack_lut_kernel, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace ob
