// linear_stack_i8.cu -- a list of one- or two-token sign-product layers in one persistent
// launch, on int8 tensor cores (i8_block.cuh).
//
// Each layer is  Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T  ("1bit量化", blog.zerodtree.com,
// "proposition 1"); a decoder applies such layers one after another.  The list is
// walked by one cooperative grid (one CTA per SM), as in linear_stack.cu, with the
// layers between two grid barriers (a barrier group) run back to back.
//
//  * Work split.  A group's rows, in 16-row tiles, are cut into one contiguous range
//    per CTA, inside one layer when the group has no more layers than CTAs (cta_range);
//    a CTA walks its range in segments (one layer, at most kMaxTiles tiles and
//    kWBufBytes of packed signs each).
//  * Weights.  A segment's packed rows are one contiguous block of memory; the CTA
//    fetches it into shared memory with one bulk copy (completion on an mbarrier).
//    Weights do not depend on activations, so the copy of the next segment is issued
//    as soon as the current one's multiply has finished with the buffer: before the
//    epilogue, and before the grid barrier when the next segment is in the next group.
//  * Activations.  After the barrier the CTA stages the segment's activation limbs
//    (i8_block.cuh) once per layer, for all its tiles.
//  * Multiply.  The eight warps take the super-blocks (512 k) of every tile of the
//    segment round robin (super-block s goes to warp s mod 8), keep exact int32 sums per
//    bit position, and fold them into per-warp fp32 tile sums in shared memory; the
//    epilogue adds those in warp order (deterministic), adds the sum of x', applies a and
//    stores.
//  * The barrier is the bounded grid barrier of stack_common.cuh; the copy waits are
//    bounded mbarrier waits.  Either running out records OB_ERR_DEVICE_TIMEOUT and ends
//    the launch.
//  * Dataflow launches (p.dataflow, one token, lists whose layers each write their own
//    buffer): no grid barrier.  A layer whose output a later layer reads also stores it as
//    32-bit words kTagMark | bf16 bits in a tag area the host zeroed before the launch; the
//    consumer's staging polls those words (bounded, with back-off) until all of its pairs'
//    words carry the mark, so it starts as soon as its own input is complete, one L2 round
//    trip after the last producer's store instead of a barrier and a load.
#include <algorithm>
#include <cstring>

#include "i8_block.cuh"
#include "stack_common.cuh"

namespace ob {
namespace {

using namespace i8;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTiles = 10;                  // tiles per segment (per-warp sums in shared memory)
constexpr uint32_t kWBufBytes = 80 * 1024;     // packed signs of one segment
constexpr int kMaxPairs = 3;                   // staging pairs per warp and chunk
constexpr int kOutPerThread = (kMaxTiles * 16 * kMaxTok + kThreads - 1) / kThreads;  // epilogue outputs
// The thread that issues the weight copies: the last one, which has no epilogue output in
// the first pass for one token, so a copy request never delays the epilogue.
constexpr int kCopyThread = kThreads - 1;

// Staged super-blocks per chunk: 22 (11 264 k, the 7B down projection in one chunk) for one
// token, 12 for two (three staging pairs per warp); with the weight buffer, the per-warp tile
// sums and the layer tables this stays inside the 227 KB a CTA may use.
template <int TOK>
constexpr int chunk_max() { return TOK == 1 ? 22 : kMaxPairs * kWarps / TOK; }

constexpr size_t red_bytes() { return sizeof(float) * kMaxTiles * kWarps * 4 * 32; }

__host__ __device__ __forceinline__ int64_t tiles_of(int64_t N) { return (N + 15) / 16; }

// The walk over the list, computed once per launch into shared memory: per layer its 16-row
// tiles, the tiles of one segment and the tiles of the earlier layers of its barrier group;
// per group its first layer and this CTA's range of its tiles.  Recomputing these between
// two grid barriers (loops over layers, divisions, parameter reads with a changing index)
// measured about a microsecond on the critical path of every group.
struct Sched {
  int32_t* tiles;  // [n_layers]
  int32_t* tpb;    // [n_layers] tiles per segment (they fit the weight buffer)
  int32_t* base;   // [n_layers] tiles of the earlier layers of the group
  int32_t* gs;     // [n_groups + 1] first layer of each group, then n_layers
  int32_t* lo;     // [n_groups] this CTA's range of group tiles [lo, hi)
  int32_t* hi;
  int ng;          // groups
};

// The range [lo, hi) of group tiles (the group's layers' tiles concatenated) that CTA c of
// G owns, for the group of layers [l, e) (tile counts and T < 2^31: checked on the host).
// When the group has no more layers than CTAs, every layer gets a contiguous set of CTAs
// in proportion to its tiles (at least one), and a CTA's range stays inside one layer: no
// CTA stages two layers' activations or waits for a second weight copy while the others are
// done.  Otherwise the concatenated tiles are cut evenly.
__device__ void cta_range(const int32_t* tiles, int l, int e, int c, int G, int32_t* lo, int32_t* hi) {
  int64_t T = 0;
  for (int li = l; li < e; ++li) T += tiles[li];
  const int nl = e - l;
  if (nl > G) {
    *lo = (int32_t)(T * c / G);
    *hi = (int32_t)(T * (c + 1) / G);
    return;
  }
  int64_t before = 0;  // tiles of the layers before li
  for (int li = l; li < e; ++li) {
    const int64_t Ti = tiles[li];
    const int i = li - l;
    // c < c1 = floor((G - nl)(before + Ti) / T) + i + 1  <=>  (c - i) T <= (G - nl)(before + Ti)
    if ((int64_t)(c - i) * T <= (int64_t)(G - nl) * (before + Ti)) {
      const int c0 = (int)((int64_t)(G - nl) * before / T) + i;
      const int c1 = (int)((int64_t)(G - nl) * (before + Ti) / T) + i + 1;
      const int64_t gi = c1 - c0, k = c - c0;
      *lo = (int32_t)(before + Ti * k / gi);
      *hi = (int32_t)(before + Ti * (k + 1) / gi);
      return;
    }
    before += Ti;
  }
  *lo = *hi = (int32_t)T;
}

struct Seg {
  int layer;   // -1: none
  int64_t t0;  // first tile within the layer
  int nt;      // tiles
};

// Tiles of one segment that fit the weight buffer for a layer of kw packed words per row.
__device__ __forceinline__ int tiles_per_buffer(int64_t kw) {
  const int64_t per_tile = 16 * 4 * kw;
  return (int)min64(kMaxTiles, max((int64_t)1, (int64_t)kWBufBytes / per_tile));
}

// The segment of group gi that starts at group tile `pos` (lo <= pos < hi).
__device__ __forceinline__ Seg seg_at(const Sched& sc, int gi, int64_t pos) {
  const int e = sc.gs[gi + 1];
  for (int li = sc.gs[gi]; li < e; ++li) {
    const int64_t base = sc.base[li], nt = sc.tiles[li];
    if (pos < base + nt) {
      const int64_t end = min((int64_t)sc.hi[gi], base + nt);
      return Seg{li, pos - base, (int)min64(end - pos, sc.tpb[li])};
    }
  }
  return Seg{-1, 0, 0};
}

// The first segment this CTA computes in group gi or a later one (groups where its range is
// empty are skipped).
__device__ __forceinline__ Seg first_seg(const Sched& sc, int gi) {
  for (; gi < sc.ng; ++gi)
    if (sc.lo[gi] < sc.hi[gi]) return seg_at(sc, gi, sc.lo[gi]);
  return Seg{-1, 0, 0};
}

// One thread: request the scale vectors of segment s (of layer L) into L2: the input scale
// is read by the staging right after a grid barrier, the output scale by the epilogue.
__device__ void prefetch_scales(const StackLayer& L, const Seg& s) {
  const int64_t r0 = s.t0 * 16, r1 = min64((s.t0 + s.nt) * 16, L.N);
  if (L.iscale)
    for (int64_t off = 0; off < L.K * 4; off += 4096) prefetch_l2_bulk(reinterpret_cast<const char*>(L.iscale) + off,
                                                                      (uint32_t)min64(4096, L.K * 4 - off));
  prefetch_l2_bulk(L.oscale + r0, (uint32_t)((r1 - r0) * 4));
}

// One thread: request the packed rows of segment s (of layer L) into the buffer.  The bulk
// copy takes the largest multiple of 16 bytes; the at most three words after it are copied
// by this thread first, so that the arrival (a release) publishes them with the phase.
// Every earlier read of the buffer has completed (a CTA barrier precedes every call); the
// proxy fence orders those generic-proxy reads before the copy's asynchronous writes.
__device__ void fetch_seg(const StackLayer& L, const Seg& s, uint32_t* wbuf, uint64_t* bar) {
  const int64_t Wd = L.K / 32;
  const int64_t r0 = s.t0 * 16, r1 = min64((s.t0 + s.nt) * 16, L.N);
  const uint64_t words = (uint64_t)((r1 - r0) * Wd);
  const uint32_t bulk = (uint32_t)(words * 4u) & ~15u;
  const uint32_t* src = L.S + r0 * Wd;
  for (uint64_t w = bulk / 4u; w < words; ++w) wbuf[w] = __ldg(src + w);
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(bar, bulk);
  if (bulk) bulk_g2s(wbuf, src, bulk, bar);
  prefetch_scales(L, s);
}

// The last warp copies layer li's descriptor from the parameter block into shared memory
// (22 words, one per lane).  The caller makes the copy visible (a CTA barrier, or
// __syncwarp for the same warp) before it is read.
static_assert(sizeof(StackLayer) == 88, "a layer descriptor is 22 words");
__device__ __forceinline__ void load_desc(const StackParams& p, int li, StackLayer* dst, int lane) {
  if (lane < 22) reinterpret_cast<uint32_t*>(dst)[lane] = reinterpret_cast<const uint32_t*>(&p.L[li])[lane];
}

// Packed words of row `row` (relative to the segment) for a super-block: words w0 .. w0+3.
// Rows at or past nrows, and words past Wd, read as zero.
__device__ __forceinline__ uint4 smem_words(const uint32_t* wbuf, int64_t Wd, int64_t row, int64_t nrows,
                                            int64_t w0, bool vec) {
  uint4 r = make_uint4(0u, 0u, 0u, 0u);
  if (row >= nrows || w0 >= Wd) return r;
  const uint32_t* q = wbuf + row * Wd + w0;
  if (vec) return *reinterpret_cast<const uint4*>(q);
  r.x = q[0];
  if (w0 + 1 < Wd) r.y = q[1];
  if (w0 + 2 < Wd) r.z = q[2];
  if (w0 + 3 < Wd) r.w = q[3];
  return r;
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 1) sign_stack_i8_kernel(const __grid_constant__ StackParams p, int ch) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ float tsum[TOK];
  __shared__ __align__(8) uint64_t wbar;
  __shared__ __align__(8) StackLayer s_desc[2];  // descriptors of the current and the next segment
  __shared__ int32_t s_tiles[kStackMaxLayers], s_tpb[kStackMaxLayers], s_base[kStackMaxLayers];
  __shared__ int32_t s_gs[kStackMaxLayers + 1], s_lo[kStackMaxLayers], s_hi[kStackMaxLayers];
  __shared__ int s_ng;
  __shared__ int s_ok;
  __shared__ int s_abort;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const bool copier_warp = warp == kWarps - 1;
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(dsm);
  const Stage<TOK> st = Stage<TOK>::carve(dsm + kWBufBytes, ch);
  float* red = reinterpret_cast<float*>(dsm + kWBufBytes + ((Stage<TOK>::bytes(ch) + 127) & ~(size_t)127));
  // The schedule: per-layer numbers, the group starts (a ballot scan by warp 0), then each
  // thread one group: the tiles before each of its layers and this CTA's range.
  for (int li = tid; li < p.n; li += kThreads) {
    s_tiles[li] = (int32_t)tiles_of(p.L[li].N);
    s_tpb[li] = tiles_per_buffer(p.L[li].K / 32);
  }
  if (warp == 0) {
    int cnt = 0;
    for (int b0 = 0; b0 < p.n; b0 += 32) {
      const int li = b0 + lane;
      const bool start = li < p.n && (li == 0 || p.L[li].barrier);
      const unsigned mask = __ballot_sync(0xffffffffu, start);
      if (start) s_gs[cnt + __popc(mask & ((1u << lane) - 1u))] = li;
      cnt += __popc(mask);
    }
    if (lane == 0) {
      s_gs[cnt] = p.n;
      s_ng = cnt;
    }
  }
  __syncthreads();
  for (int g = tid; g < s_ng; g += kThreads) {
    const int gl = s_gs[g], ge = s_gs[g + 1];
    int32_t before = 0;
    for (int li = gl; li < ge; ++li) {
      s_base[li] = before;
      before += s_tiles[li];
    }
    cta_range(s_tiles, gl, ge, c, G, &s_lo[g], &s_hi[g]);
  }
  const Sched sc{s_tiles, s_tpb, s_base, s_gs, s_lo, s_hi, 0};
  if (tid == 0) {
    mbar_init(&wbar, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();
  pdl_wait();  // the first layers' inputs may come from the previous grid in the stream

  uint32_t wphase = 0;    // completed weight copies
  int staged = -1;        // layer whose activation limbs are staged (single chunk only)
  Seg pending{-1, 0, 0};  // segment whose copy is in flight (its descriptor in s_desc[cur])
  int cur = 0;

  const int ng = s_ng;
  Sched scg = sc;
  scg.ng = ng;
  {
    const Seg s0 = first_seg(scg, 0);
    if (s0.layer >= 0 && copier_warp) {
      load_desc(p, s0.layer, &s_desc[cur], lane);
      __syncwarp();
      if (tid == kCopyThread) {
        fetch_seg(s_desc[cur], s0, wbuf, &wbar);
        const Seg s1 = first_seg(scg, 1);  // the second group's scales (later ones: at the barriers)
        if (s1.layer >= 0) prefetch_scales(p.L[s1.layer], s1);
      }
    }
    pending = s0;
  }
  unsigned barriers = 0;
  for (int gi = 0; gi < ng; ++gi) {
    const int64_t hi = s_hi[gi];
    for (int64_t pos = s_lo[gi]; pos < hi;) {
      const Seg sg = seg_at(scg, gi, pos);
      __syncthreads();  // the previous segment's epilogue no longer reads red / tsum; s_desc[cur] is written
      if (pending.layer != sg.layer || pending.t0 != sg.t0 || pending.nt != sg.nt) {
        // Not the segment requested ahead (the walk above always requests this one; kept
        // for safety): let any stray copy land, then request this one.
        if (pending.layer >= 0) {
          mbar_wait(&wbar, wphase & 1u, p.err, &s_abort);
          ++wphase;
        }
        if (copier_warp) {
          load_desc(p, sg.layer, &s_desc[cur], lane);
          __syncwarp();
          if (tid == kCopyThread) fetch_seg(s_desc[cur], sg, wbuf, &wbar);
        }
        __syncthreads();
      }
      pending = Seg{-1, 0, 0};
      const StackLayer& L = s_desc[cur];
      SignGemmArgs g{L.X, p.M, L.K, L.S, L.N, L.iscale, L.oscale, L.Y, L.N, L.y_dtype, 0};
      const int64_t K = L.K, Wd = K / 32, nsb = (K + kSbK - 1) / kSbK;
      const int64_t mt = min64(TOK, p.M);
      const int64_t nrows = min64(sg.nt * 16, L.N - sg.t0 * 16);
      const bool single_chunk = nsb <= ch;
      // The output scales this thread's epilogue applies, requested now so that their latency
      // is hidden by the staging and the multiply.
      float osc[kOutPerThread];
#pragma unroll
      for (int j = 0; j < kOutPerThread; ++j) {
        const int idx = tid + j * kThreads;
        const int r = idx % (sg.nt * 16);
        osc[j] = (idx < sg.nt * 16 * TOK && r < nrows) ? __ldg(L.oscale + sg.t0 * 16 + r) : 0.f;
      }
      for (int64_t sb0 = 0; sb0 < nsb; sb0 += ch) {
        const int chn = (int)min64(ch, nsb - sb0);
        if (!(single_chunk && staged == sg.layer)) {
          // Earlier readers of the stage and of tsum are done: the barrier at the top of the
          // segment (first chunk) or the one after the previous chunk's multiply.
          // Staging: the pairs (token, super-block) p = warp, warp + 8, warp + 16, each with
          // its own scale; then warp 7 sums T while the others start multiplying.
          StageRaw raw[kMaxPairs];
          if (L.tag_in) {
            // Dataflow: the input is an earlier layer's tagged output; poll the pairs' words
            // until every one carries the mark (the area was zeroed before the launch).
            bool in_ok = true;
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t it = 0;; ++it) {
              bool ready = true;
#pragma unroll
              for (int k = 0; k < kMaxPairs; ++k) {
                const int pp = warp + k * kWarps;
                if (pp < TOK * chn)
                  ready &= stage_load_tagged(g, L.tag_in, pp % TOK, pp % TOK < mt, (sb0 + pp / TOK) * kSbK, lane,
                                             raw[k]);
              }
              if (__all_sync(0xffffffffu, ready)) break;
              if ((it & 15u) == 15u) {
                if (ld_acquire_gpu(p.bar + 1) != 0u) {
                  in_ok = false;
                  break;
                }
                if (globaltimer_ns() - t0 > OB_WAIT_LIMIT_NS || it > (1u << 24)) {
                  if (lane == 0) {
                    record_error(p.err, OB_DEVERR_TIMEOUT);
                    atomicExch(p.bar + 1, 1u);
                  }
                  in_ok = false;
                  break;
                }
              }
              __nanosleep(it < 4 ? 64 : 256);
            }
            if (!in_ok && lane == 0) s_abort = 1;
          } else {
#pragma unroll
            for (int k = 0; k < kMaxPairs; ++k) {
              const int pp = warp + k * kWarps;
              if (pp < TOK * chn) raw[k] = stage_load<true>(g, pp % TOK, pp % TOK < mt, (sb0 + pp / TOK) * kSbK, lane);
            }
          }
#pragma unroll
          for (int k = 0; k < kMaxPairs; ++k) {
            const int pp = warp + k * kWarps;
            if (pp < TOK * chn) stage_pair<TOK>(raw[k], pp % TOK, st, pp / TOK, lane);
          }
          __syncthreads();
          if (warp == kWarps - 1) {
#pragma unroll
            for (int m = 0; m < TOK; ++m) {
              const float t = chunk_sum<TOK>(st, chn, m, lane);
              if (lane == 0) tsum[m] = (sb0 == 0 ? 0.f : tsum[m]) + t;
            }
          }
          staged = single_chunk ? sg.layer : -1;
        }
        if (sb0 == 0) {  // this segment's weights
          if (!mbar_wait(&wbar, wphase & 1u, p.err, &s_abort)) {
            s_abort = 1;
            // One more bounded wait, so that no copy is left in flight at exit.
            mbar_wait(&wbar, wphase & 1u, p.err, nullptr);
          }
          ++wphase;
        }
        // Multiply: warp w takes super-blocks w, w + 8, ... of the chunk for every tile,
        // with exact int32 sums per bit position, folded into the warp's tile sums.  A warp
        // without a super-block in the first chunk writes zeros.
        if (!s_abort && chn <= kWarps) {
          // At most one super-block per warp (K <= 4096 in one chunk): its fragments stay in
          // registers for all the tiles, and each tile's words are requested one tile ahead.
          const int s = warp;
          const float f0 = s < chn ? st.fold_at(s)[2 * tq] : 0.f, f1 = s < chn ? st.fold_at(s)[2 * tq + 1] : 0.f;
          SbRegs fr;
          if (s < chn) load_sb_regs(st.frag_at(s), lane, fr);
          const int64_t w0 = (sb0 + s) * kSbWords + 4 * tq;
          uint4 wg = make_uint4(0u, 0u, 0u, 0u), wh = wg;
          if (s < chn) {
            wg = smem_words(wbuf, Wd, gq, nrows, w0, L.vec != 0);
            wh = smem_words(wbuf, Wd, gq + 8, nrows, w0, L.vec != 0);
          }
          for (int i = 0; i < sg.nt; ++i) {
            uint4 ng = make_uint4(0u, 0u, 0u, 0u), nh = ng;
            if (s < chn && i + 1 < sg.nt) {
              ng = smem_words(wbuf, Wd, 16 * (i + 1) + gq, nrows, w0, L.vec != 0);
              nh = smem_words(wbuf, Wd, 16 * (i + 1) + gq + 8, nrows, w0, L.vec != 0);
            }
            int acc[kChains][4];
#pragma unroll
            for (int j = 0; j < kChains; ++j)
#pragma unroll
              for (int r = 0; r < 4; ++r) acc[j][r] = 0;
            if (s < chn) tile_sb_regs(fr, wg, wh, acc);
            float* dst = red + (size_t)(i * kWarps + warp) * 128;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float v = (float)combine(acc, r) * ((r & 1) ? f1 : f0);
              float* d = dst + r * 32 + lane;
              *d = sb0 == 0 ? v : *d + v;
            }
            wg = ng;
            wh = nh;
          }
        } else if (!s_abort) {
          for (int i = 0; i < sg.nt; ++i) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            for (int s = warp; s < chn; s += kWarps) {
              int acc[kChains][4];
#pragma unroll
              for (int j = 0; j < kChains; ++j)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[j][r] = 0;
              const int64_t w0 = (sb0 + s) * kSbWords + 4 * tq;
              const uint4 wg = smem_words(wbuf, Wd, 16 * i + gq, nrows, w0, L.vec != 0);
              const uint4 wh = smem_words(wbuf, Wd, 16 * i + gq + 8, nrows, w0, L.vec != 0);
              tile_sb(st.frag_at(s), wg, wh, acc, lane);
              const float* f = st.fold_at(s);
              const float f0 = f[2 * tq], f1 = f[2 * tq + 1];
#pragma unroll
              for (int r = 0; r < 4; ++r) v[r] = fmaf((float)combine(acc, r), (r & 1) ? f1 : f0, v[r]);
            }
            float* dst = red + (size_t)(i * kWarps + warp) * 128;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              float* d = dst + r * 32 + lane;
              *d = sb0 == 0 ? v[r] : *d + v[r];
            }
          }
        }
        __syncthreads();  // multiply done: the weight buffer and this chunk's stage are free
      }
      if (s_abort) return;
      // Request the next segment's weights (this group's next, or the next group's first),
      // with its descriptor in the other slot.
      pos += sg.nt;
      pending = pos < hi ? seg_at(scg, gi, pos) : first_seg(scg, gi + 1);
      if (pending.layer >= 0 && copier_warp) {
        load_desc(p, pending.layer, &s_desc[cur ^ 1], lane);
        __syncwarp();
        if (tid == kCopyThread) fetch_seg(s_desc[cur ^ 1], pending, wbuf, &wbar);
      }
      // Epilogue: sum the warps' tile sums, add T, scale (loaded above), store.
#pragma unroll
      for (int j = 0; j < kOutPerThread; ++j) {
        const int idx = tid + j * kThreads;
        if (idx >= sg.nt * 16 * TOK) break;
        const int r = idx % (sg.nt * 16), m = idx / (sg.nt * 16);
        const int64_t n = sg.t0 * 16 + r;
        if (m >= mt || r >= nrows) continue;
        const int i = r >> 4, r16 = r & 15;
        const int gg = r16 & 7, hh = r16 >> 3;
        float v = tsum[m];
#pragma unroll
        for (int li = 0; li < kLimbs; ++li) {
          const int col = kLimbs * m + li;
          const int src = 4 * gg + (col >> 1), reg = 2 * hh + (col & 1);
          for (int w = 0; w < kWarps; ++w) v += red[(size_t)(i * kWarps + w) * 128 + reg * 32 + src];
        }
        v *= osc[j];
        const int64_t off = (int64_t)m * L.N + n;
        if (L.y_dtype == OB_OUT_F32) {
          static_cast<float*>(L.Y)[off] = v;
        } else {
          const __nv_bfloat16 yb = __float2bfloat16_rn(v);
          static_cast<__nv_bfloat16*>(L.Y)[off] = yb;
          if (L.tag_out) st_volatile_u32(L.tag_out + off, kTagMark | (uint32_t)__bfloat16_as_ushort(yb));
        }
      }
      cur ^= 1;
    }
    staged = -1;  // the next group's inputs are new
    // Dataflow launches have no grid barrier: a consumer polls its producer's tagged output.
    if (gi + 1 < ng && !p.dataflow) {
      ++barriers;
      // While thread 0 waits, the copy thread requests the scale vectors of the group after
      // the next into L2 (the next group's were requested with its weights, which is late for
      // the input scale its staging reads first).
      const auto side = [&]() {
        if (tid == kCopyThread) {
          const Seg a = first_seg(scg, gi + 2);
          if (a.layer >= 0) prefetch_scales(p.L[a.layer], a);
        }
      };
      if (!grid_barrier(p.bar, barriers * (unsigned)G, p.err, &s_ok, side)) {
        // Leave no bulk copy in flight into this CTA's shared memory.
        if (pending.layer >= 0) mbar_wait(&wbar, wphase & 1u, p.err, nullptr);
        return;
      }
    }
  }
}

template <int TOK>
cudaError_t launch_i8_tok(const StackParams& prm, const LaunchCtx& c) {
  auto kern = sign_stack_i8_kernel<TOK>;
  int64_t max_k = 32;
  for (int i = 0; i < prm.n; ++i) max_k = std::max<int64_t>(max_k, prm.L[i].K);
  const int ch = (int)std::min<int64_t>(chunk_max<TOK>(), (max_k + kSbK - 1) / kSbK);
  const size_t smem = kWBufBytes + ((Stage<TOK>::bytes(ch) + 127) & ~(size_t)127) + red_bytes();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
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

bool stack_i8_supported(const StackParams& prm) {
  if (prm.M > kMaxTok) return false;
  int64_t group = 0;  // tiles of the current barrier group (kept in 32-bit shared-memory tables)
  for (int i = 0; i < prm.n; ++i) {
    if (16 * (prm.L[i].K / 8) > (int64_t)kWBufBytes) return false;  // one tile must fit the weight buffer
    if (i > 0 && prm.L[i].barrier) group = 0;
    group += tiles_of(prm.L[i].N);
    if (group >= ((int64_t)1 << 31)) return false;
  }
  return true;
}

cudaError_t launch_stack_i8(const StackParams& prm, const LaunchCtx& c) {
  return prm.M == 1 ? launch_i8_tok<1>(prm, c) : launch_i8_tok<2>(prm, c);
}

}  // namespace ob
