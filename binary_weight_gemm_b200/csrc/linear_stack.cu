// linear_stack.cu -- a list of small-M sign-product layers in one persistent launch.
//
// Each layer is  Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T  ("1bit量化", blog.zerodtree.com,
// "proposition 1"); a decoder applies such layers one after another, a layer
// reading the output of an earlier one.  Launched one kernel per layer, every
// dependent layer pays a launch and a drain; here one cooperative grid walks the
// whole list.  This file holds the bf16 warp-level MMA form (any M <= 16) and the
// launcher, which takes the int8 form of linear_stack_i8.cu for one or two tokens.
// The bf16 MMA form:
//  * A layer flagged as reading an earlier layer's output waits at a grid-wide
//    barrier; the layers between two barriers run back to back.
//  * A layer's rows are split into 32-row blocks dealt to the CTAs round robin,
//    continuing across the layers of one barrier group, so independent layers
//    (q, k, v) spread over the whole grid.  A block is the warp-level MMA block of
//    the decode kernel (mma_decode_block.cuh), reading activations through L2
//    (other CTAs of this grid wrote them).
//  * Weights do not depend on activations: before computing a group, each CTA
//    prefetches into L2 the sign rows of its blocks of the next group, so they
//    stream in while this group computes and while the grid waits at the barrier.
//  * The barrier is a counter in the caller's workspace (zeroed before the launch);
//    its wait is bounded: a CTA that gives up records a timeout in the error
//    word and sets an abort word that makes every other CTA leave at its next barrier.
#include <algorithm>
#include <vector>
#include <cstring>

#include "mma_decode_block.cuh"
#include "stack_common.cuh"

namespace ob {
namespace {

using namespace mmad;

// First block of a layer dealt to CTA c when the group's round robin is at `off`.
__device__ __forceinline__ int first_block(int c, int off, int G) {
  const int t = c - off;
  return t < 0 ? t + G : t;
}

// Prefetch into L2 what this CTA reads of layers [l, e): the sign rows of its
// blocks and the layers' scale vectors, given the round-robin offset `off` of the
// group.  Called by one warp.
__device__ void prefetch_group(const StackParams& p, int l, int e, int off, int lane) {
  const int G = gridDim.x, c = blockIdx.x;
  for (int li = l; li < e; ++li) {
    const StackLayer& L = p.L[li];
    const int64_t Wd = L.K / 32;
    for (int t = first_block(c, off, G); t < L.nb; t += G) {
      const int64_t r0 = (int64_t)t * kRowsPerCta, rows = min64(kRowsPerCta, L.N - r0);
      if (((r0 * Wd) & 3) == 0 && (reinterpret_cast<uintptr_t>(L.S) & 15) == 0)
        prefetch_block_l2(L.S + r0 * Wd, (uint64_t)(rows * Wd) * 4u, lane);
    }
    if (L.iscale) prefetch_block_l2(L.iscale, (uint64_t)L.K * 4u, lane);
    prefetch_block_l2(L.oscale, (uint64_t)L.N * 4u, lane);
    off = (off + L.nb) % G;
  }
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 1) sign_stack_kernel(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ BlockShared<TOK> shb;
  __shared__ int s_ok;
  const int G = gridDim.x, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int e = group_end(p, 0);
  if (warp == 0) prefetch_group(p, 0, e, 0, lane);
  pdl_wait();  // the first layers' inputs may come from the previous grid in the stream
  unsigned barriers = 0;
  int off = 0;
  for (int l = 0; l < p.n;) {
    // Sum of this group's blocks: the round-robin offset of the next group.
    int next_off = off;
    for (int li = l; li < e; ++li) next_off = (next_off + p.L[li].nb) % G;
    const int e2 = e < p.n ? group_end(p, e) : e;
    if (warp == 0 && e < p.n) prefetch_group(p, e, e2, next_off, lane);
    for (int li = l; li < e; ++li) {
      const StackLayer& L = p.L[li];
      SignGemmArgs g{L.X, p.M, L.K, L.S, L.N, L.iscale, L.oscale, L.Y, L.N, L.y_dtype, 0};
      for (int t = first_block(c, off, G); t < L.nb; t += G)
        block<TOK, true>(g, 0, (int64_t)t * kRowsPerCta, L.vec != 0, dsm, shb);
      off = (off + L.nb) % G;
    }
    l = e;
    e = e2;
    if (l < p.n) {
      ++barriers;
      if (!grid_barrier(p.bar, barriers * (unsigned)G, p.err, &s_ok)) return;
    }
  }
}

template <int TOK>
cudaError_t launch_stack_tok(const StackParams& prm, const LaunchCtx& c) {
  auto kern = sign_stack_kernel<TOK>;
  const size_t smem = dyn_smem_bytes<TOK>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
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
  e = cudaLaunchKernelEx(&cfg, kern, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int stack_max_layers_per_launch() { return kStackMaxLayers; }

namespace {

// The dataflow plan of one launch's layers [0, n): producer of each layer's input (-1: an
// input from outside the launch) and tag offsets (words; -1: no consumer).  Returns the tag
// words needed, or -1 when the launch does not qualify (an output overlaps another output,
// or an input that is not exactly an earlier layer's bf16 output).
int64_t dataflow_plan(const StackLayerHost* L, int n, int64_t M, std::vector<int>& prod, std::vector<int64_t>& off) {
  prod.assign((size_t)n, -1);
  off.assign((size_t)n, -1);
  auto ybytes = [&](int i) { return (uintptr_t)(M * L[i].N * (L[i].y_dtype == OB_OUT_F32 ? 4 : 2)); };
  auto xbytes = [&](int i) { return (uintptr_t)(M * L[i].K * 2); };
  auto overlap = [](uintptr_t a, uintptr_t an, uintptr_t b, uintptr_t bn) { return a < b + bn && b < a + an; };
  for (int j = 0; j < n; ++j) {
    const uintptr_t xj = reinterpret_cast<uintptr_t>(L[j].X), yj = reinterpret_cast<uintptr_t>(L[j].Y);
    for (int i = j - 1; i >= 0 && prod[j] < 0; --i)
      if (reinterpret_cast<uintptr_t>(L[i].Y) == xj && L[i].y_dtype == OB_OUT_BF16 && ybytes(i) == xbytes(j))
        prod[j] = i;
    for (int i = 0; i < n; ++i) {
      const uintptr_t yi = reinterpret_cast<uintptr_t>(L[i].Y);
      if (i != j && overlap(yi, ybytes(i), yj, ybytes(j))) return -1;          // two layers write one buffer
      if (overlap(yi, ybytes(i), xj, xbytes(j)) && i != prod[j]) return -1;    // not a producer's output
    }
  }
  // Each tagged output starts on a 256-byte boundary: consumers read it 16 bytes at a time.
  int64_t words = 0;
  for (int j = 0; j < n; ++j)
    if (prod[j] >= 0 && off[(size_t)prod[j]] < 0) {
      off[(size_t)prod[j]] = words;
      words += (M * L[prod[j]].N + 63) & ~(int64_t)63;
    }
  return words;
}

}  // namespace

size_t stack_tag_words(const StackLayerHost* layers, int n, int64_t M) {
  // One token: on the 7B stack the dataflow form measured 1018 against 1191 us per token with
  // barriers; at two tokens 1403 against 1368 us per step, so two tokens keep the barriers.
  if (M != 1) return 0;
  size_t most = 0;
  std::vector<int> prod;
  std::vector<int64_t> off;
  for (int base = 0; base < n; base += kStackMaxLayers) {
    const int cnt = std::min(kStackMaxLayers, n - base);
    const int64_t w = dataflow_plan(layers + base, cnt, M, prod, off);
    if (w < 0) return 0;  // one launch of the list would need barriers: no dataflow for the list
    most = std::max(most, (size_t)w);
  }
  return most;
}

cudaError_t launch_sign_stack(const StackLayerHost* layers, int n, int64_t M, unsigned* bar, const LaunchCtx& c,
                              int path, uint32_t* tags, size_t tag_words) {
  if (n == 0 || M == 0) return cudaSuccess;
  static_assert(sizeof(StackParams) <= 32000, "kernel parameters");
  StackParams* prm = new StackParams;
  std::memset(prm, 0, sizeof(StackParams));
  cudaError_t e = cudaSuccess;
  std::vector<int> prod;
  std::vector<int64_t> off;
  for (int base = 0; base < n && e == cudaSuccess; base += kStackMaxLayers) {
    const int cnt = std::min(kStackMaxLayers, n - base);
    prm->n = cnt;
    prm->M = M;
    prm->bar = bar;
    prm->err = c.err;
    for (int i = 0; i < cnt; ++i) {
      const StackLayerHost& h = layers[base + i];
      const int nb = (int)((h.N + kRowsPerCta - 1) / kRowsPerCta);
      const int vec = ((h.K / 32) % 4 == 0) && ((reinterpret_cast<uintptr_t>(h.S) & 15) == 0);
      prm->L[i] = StackLayer{static_cast<const uint16_t*>(h.X), h.S, h.iscale, h.oscale, h.Y, h.K, h.N, h.y_dtype,
                             i == 0 ? 0 : h.barrier, nb, vec, nullptr, nullptr};
    }
    const bool i8 = path == OB_PATH_I8 && stack_i8_supported(*prm);
    // Dataflow: the int8 form, a tag area, and a launch that qualifies.
    int64_t words = -1;
    if (i8 && tags && M == 1) words = dataflow_plan(layers + base, cnt, M, prod, off);
    prm->dataflow = (words >= 0 && (size_t)words <= tag_words) ? 1 : 0;
    if (prm->dataflow)
      for (int i = 0; i < cnt; ++i) {
        if (off[(size_t)i] >= 0) prm->L[i].tag_out = tags + off[(size_t)i];
        if (prod[(size_t)i] >= 0) prm->L[i].tag_in = tags + off[(size_t)prod[(size_t)i]];
      }
    e = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned), c.stream);
    if (e == cudaSuccess && prm->dataflow && words > 0)
      e = cudaMemsetAsync(tags, 0, (size_t)words * sizeof(uint32_t), c.stream);  // no word is ready yet
    if (e != cudaSuccess) break;
    if (i8)
      e = launch_stack_i8(*prm, c);
    else
      e = M == 1 ? launch_stack_tok<1>(*prm, c) : (M <= 8 ? launch_stack_tok<8>(*prm, c) : launch_stack_tok<16>(*prm, c));
  }
  delete prm;
  return e;
}

}  // namespace ob
