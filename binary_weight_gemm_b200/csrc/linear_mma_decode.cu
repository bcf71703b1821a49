// linear_mma_decode.cu -- small-M sign product with warp-level tensor-core MMA.
//
//   Y[m, n] = oscale[n] * sum_k (x[m, k] * iscale[k]) * s[n, k],   M <= 16 per pass
//
// "1bit量化" (blog.zerodtree.com), "proposition 1": Y = [(X ⊙ b^T) W_sign^T] ⊙ a^T;
// each of DBF's two sign products ("Addition is almost all you need ...",
// "Methodologie") is one call.
//
// Why warp-level MMA here: at decode sizes a layer is a few MB and the kernel is
// bound by latency, not by tensor throughput.  The tensor-memory path
// (tcgen05.mma from one issuing thread, tcgen05.st/ld, mbarrier and cluster
// hand-offs) adds latency that N <= 16 cannot amortise; mma.sync is an ordinary
// warp instruction that keeps the operands in registers.
//
// Mapping (mma.sync.m16n8k16, bf16 in, fp32 accumulate):
//  * A (16 x 16) = 16 weight rows x 16 k of +/-bf16(iscale[k]), expanded in
//    registers from the packed words with the input scale folded in
//    ((X ⊙ b) S^T = X (S ⊙ 1 b^T)^T).  The fragment's k order is permuted so that
//    each 32-bit A register pairs column c with column c+16 of one packed word:
//    ((w << (15-c)) & 0x80008000) ^ bf16x2(b_c, b_c+16), one shift and one LOP3
//    for two weights.  Fragment position p of k-step s of word w is
//    k = 32w + 8s + p/2 + 16*(p%2).
//  * B (16 x 8) = the same 16 k x 8 tokens of x (bf16, exact), copied by each
//    warp into shared memory already in fragment order and permuted the same
//    way (one byte permutation per register), so the MMA contracts matching k.
//    M <= 8 uses one n8 tile, M <= 16 two.
//  * Each tile keeps 2-4 independent accumulator sets (word w goes to set
//    w mod sets) so consecutive MMAs do not wait on each other.
//  * A CTA owns 32 weight rows (two m16 tiles); its 8 warps take 512-k chunks of
//    K round robin; partial tiles are summed across warps in shared memory, then
//    scaled by oscale and stored.
//  * Latency: before the programmatic-dependent-launch wait a CTA only prefetches
//    its sign rows into L2; after it, each warp copies its chunk's sign words
//    into shared memory with cp.async (no registers held), the next chunk's
//    words are copied while this one is computed, and each warp's activation
//    loads for a chunk are all issued before any is used.
//  * The 32-row block is a device function: one CTA per block in the per-call
//    kernel, and a persistent CTA walking a list of (layer, block) tasks in the
//    layer-stack kernel (linear_stack.cu).
#include <algorithm>

#include "ob_device.cuh"
#include "ob_internal.h"

#include "mma_decode_block.cuh"

namespace ob {
namespace {

using namespace mmad;

// TOK: tokens per pass the kernel is built for (1, 8 or 16).  One CTA per 32-row block.
template <int TOK, bool kVec>
__global__ void __launch_bounds__(kThreads, TOK > 8 ? 1 : 2) sign_gemm_mma_decode_kernel(SignGemmArgs g, int64_t m0) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ BlockShared<TOK> shb;
  const int64_t n0 = (int64_t)blockIdx.x * kRowsPerCta;
  // Before the previous grid has finished, only pull this CTA's sign rows (one
  // contiguous block) into L2; the reads themselves come after pdl_wait.  With static
  // weights (the previous grid did not write them) each warp's first chunk of sign
  // words is requested into shared memory already.
  if (g.l2_prefetch && threadIdx.x < 32 && n0 < g.R) {
    const int64_t Wd = g.K / 32;
    const int64_t rows = min64(kRowsPerCta, g.R - n0);
    prefetch_block_l2(g.S + n0 * Wd, (uint64_t)(rows * Wd) * 4u, threadIdx.x);
    if (g.iscale) prefetch_block_l2(g.iscale, (uint64_t)g.K * 4u, threadIdx.x);
  }
  if (g.static_w) fetch_words(g, n0, kVec, warp_words<TOK>(dsm, threadIdx.x >> 5), threadIdx.x >> 5, 0, threadIdx.x & 31);
  pdl_wait();  // every input may have been written by the previous grid in the stream
  pdl_launch_dependents();  // the next grid may start (one grid ahead at most)
  block<TOK, false>(g, m0, n0, kVec, dsm, shb, g.static_w != 0);
}

template <int TOK, bool kVec>
cudaError_t launch_tok(const SignGemmArgs& g, int64_t m0, const LaunchCtx& c) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((g.R + kRowsPerCta - 1) / kRowsPerCta), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  const size_t smem = dyn_smem_bytes<TOK>();
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
  auto kern = sign_gemm_mma_decode_kernel<TOK, kVec>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, kern, g, m0);
}

template <bool kVec>
cudaError_t launch_vec(const SignGemmArgs& g, int64_t m0, int64_t mt, const LaunchCtx& c) {
  if (mt == 1) return launch_tok<1, kVec>(g, m0, c);
  if (mt <= 8) return launch_tok<8, kVec>(g, m0, c);
  return launch_tok<16, kVec>(g, m0, c);
}

}  // namespace

cudaError_t launch_sign_gemm_mma_decode(const SignGemmArgs& g, const LaunchCtx& c) {
  if (g.M == 0 || g.R == 0 || g.K == 0) return cudaSuccess;
  for (int64_t m0 = 0; m0 < g.M; m0 += 16) {
    const int64_t mt = std::min<int64_t>(16, g.M - m0);
    const bool vec = ((g.K / 32) % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.S) & 15) == 0);
    cudaError_t e = vec ? launch_vec<true>(g, m0, mt, c) : launch_vec<false>(g, m0, mt, c);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace ob
