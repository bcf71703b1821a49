// pack.cu -- sign extraction and bit packing, W_sign = Sign(W).
//
// "1bit量化" (blog.zerodtree.com), section "rank-1 approximation": the weight is
// split as W = W_sign ⊙ |W| with W_sign = Sign(W); the OneBit layer keeps only
// W_±1 = Sign(W) (distillation section).  Storage format (the pages give none):
// 32 signs per uint32, rows K-major, bit i of word w <-> column 32w+i, set bit <=> -1.
//
// One warp packs 32 consecutive columns per ballot: lane i loads column 32w+i
// (128 contiguous bytes per warp load), the ballot of (w < 0) is the word.
// The kernel reads 32x the bytes it writes, so it is bound by HBM reads; each
// warp keeps several independent loads in flight.
#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kPackThreads = 256;
constexpr int kWordsPerWarpIter = 8;  // independent 128-byte loads in flight per warp

__global__ void __launch_bounds__(kPackThreads) pack_signs_kernel(const float* __restrict__ W, int64_t n_words,
                                                                  uint32_t* __restrict__ out, unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)kPackThreads + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * kPackThreads) >> 5;
  // Words are numbered over the whole matrix: word g covers elements [32g, 32g+32),
  // which equals row g / (K/32), word g % (K/32) because K is a multiple of 32.
  for (int64_t base = warp * kWordsPerWarpIter; base < n_words; base += n_warps * kWordsPerWarpIter) {
    float v[kWordsPerWarpIter];
#pragma unroll
    for (int j = 0; j < kWordsPerWarpIter; ++j) {
      const int64_t g = base + j;
      v[j] = g < n_words ? __ldcs(W + g * 32 + lane) : 1.0f;
    }
    bool any_nan = false;
#pragma unroll
    for (int j = 0; j < kWordsPerWarpIter; ++j) {
      const uint32_t word = __ballot_sync(0xffffffffu, v[j] < 0.0f);
      any_nan |= (v[j] != v[j]);
      const int64_t g = base + j;
      if (lane == j && g < n_words) out[g] = word;
    }
    if (__any_sync(0xffffffffu, any_nan) && lane == 0) record_error(err, OB_DEVERR_NAN);
  }
}

}  // namespace

cudaError_t launch_pack_signs(const float* W, int64_t N, int64_t K, uint32_t* out, const LaunchCtx& c) {
  const int64_t n_words = N * (K / 32);
  if (n_words == 0) return cudaSuccess;
  const int64_t warps_needed = (n_words + kWordsPerWarpIter - 1) / kWordsPerWarpIter;
  int64_t blocks = (warps_needed * 32 + kPackThreads - 1) / kPackThreads;
  const int64_t cap = (int64_t)c.num_sms * 8;
  if (blocks > cap) blocks = cap;
  pack_signs_kernel<<<(unsigned)blocks, kPackThreads, 0, c.stream>>>(W, n_words, out, c.err);
  return cudaGetLastError();
}

}  // namespace ob
