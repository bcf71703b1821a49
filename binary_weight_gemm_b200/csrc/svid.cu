// svid.cu -- rank-1 SVID of |W| by power iteration.
//
// "1bit量化" (blog.zerodtree.com), section "rank-1 approximation": |W| ≈ a b^T
// from the leading singular triple (u1, sigma1, v1); here a = sqrt(sigma1) u1,
// b = sqrt(sigma1) v1.  The page obtains the triple from an SVD; on the GPU the
// leading right vector is found by power iteration on the Gram matrix:
//
//     v_0 = 1/sqrt(K)                      (positive, so never orthogonal to the
//                                            nonnegative leading vector of |W|)
//     y   = |W|^T (|W| v_t),  v_{t+1} = y / ||y||
//     stop when ||v_{t+1} - v_t||_2 <= tol
//
// then z = |W| v, sigma1 = ||z||, a = z / sqrt(sigma1), b = sqrt(sigma1) v.
// Each iteration is two passes over fp32 W (a row GEMV and a column GEMV); all
// reductions are fp32 inside a thread and fp64 across threads.  The column
// GEMV writes per-split partial sums that a second kernel adds in a fixed
// order, so the iteration itself is deterministic; only the fp64 norm
// accumulators use atomics.
//
// The stopping test runs on the device: the last block of each iteration's
// update kernel decides whether the iteration converged (or met a NaN) and
// sets a flag that turns every later kernel of the loop into a no-op.  The host
// queues iterations in batches of kBatch followed by the final pass, and reads
// the outcome back once per batch: once in all, when the iteration converges
// within the first batch.
#include <algorithm>
#include <cmath>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr int kSplitsMax = 64;
constexpr int kColThreads = 256;

constexpr int kBatch = 8;  // iterations queued between two reads of the outcome

struct SvidScalars {
  double yy;         // ||y||^2 of the current iteration
  double diff2;      // ||v_new - v||^2 of the current iteration
  double zz;         // ||z||^2 in the final pass
  unsigned arrived;  // blocks of the current update kernel that have added their share
  int state;         // kRunning, kConverged or kNan
  int iters;         // iterations completed
  int pad;
};

constexpr int kRunning = 0, kConverged = 1, kNan = 2;

__device__ __forceinline__ int svid_state(const SvidScalars* sc) {
  return *reinterpret_cast<const volatile int*>(&sc->state);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct SvidLayout {
  size_t off_v, off_z, off_y, off_part, total;
  SvidLayout(int64_t N, int64_t K) {
    size_t o = align256(sizeof(SvidScalars));
    off_v = o; o = align256(o + sizeof(float) * (size_t)K);
    off_z = o; o = align256(o + sizeof(float) * (size_t)N);
    off_y = o; o = align256(o + sizeof(float) * (size_t)K);
    off_part = o; o = align256(o + sizeof(float) * (size_t)K * kSplitsMax);
    total = o;
  }
};

__global__ void svid_init_kernel(float* v, int64_t K) {
  const float v0 = rsqrtf((float)K);
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < K; k += (int64_t)gridDim.x * blockDim.x)
    v[k] = v0;
}

// z[n] = sum_k |W[n,k]| v[k]; one warp per row, float4 loads.  If zz != null,
// also accumulates ||z||^2.
// final == false: an iteration's pass, skipped once the loop has stopped.  final == true:
// the pass after the loop (zz = ||z||^2), run when it converged, or at the cap (force).
__device__ __forceinline__ bool svid_skip(const SvidScalars* sc, bool final, bool force) {
  const int st = svid_state(sc);
  return final ? !(st == kConverged || (force && st == kRunning)) : st != kRunning;
}

__global__ void __launch_bounds__(256) svid_rowdot_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                                          const float* __restrict__ v, float* __restrict__ z,
                                                          SvidScalars* sc, bool final, bool force) {
  if (svid_skip(sc, final, force)) return;
  double* zz = final ? &sc->zz : nullptr;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t K4 = K / 4;
  for (int64_t n = warp; n < N; n += n_warps) {
    const float4* row = reinterpret_cast<const float4*>(W + n * K);
    const float4* v4 = reinterpret_cast<const float4*>(v);
    float acc = 0.f;
    for (int64_t j = lane; j < K4; j += 32) {
      const float4 w = __ldcs(row + j);
      const float4 x = __ldg(v4 + j);
      acc += fabsf(w.x) * x.x + fabsf(w.y) * x.y + fabsf(w.z) * x.z + fabsf(w.w) * x.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      z[n] = acc;
      if (zz) atomicAdd(zz, (double)acc * (double)acc);
    }
  }
}

// part[s][k] = sum over rows n of split s of |W[n,k]| z[n]; one thread per column.
__global__ void __launch_bounds__(kColThreads) svid_coldot_kernel(const float* __restrict__ W, int64_t N,
                                                                   int64_t K, const float* __restrict__ z,
                                                                   float* __restrict__ part,
                                                                   int64_t rows_per_split, const SvidScalars* sc) {
  if (svid_skip(sc, false, false)) return;
  const int64_t k = blockIdx.x * (int64_t)kColThreads + threadIdx.x;
  const int64_t s = blockIdx.y;
  const int64_t n0 = s * rows_per_split;
  const int64_t n1 = min(N, n0 + rows_per_split);
  if (k >= K) return;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  int64_t n = n0;
  for (; n + 4 <= n1; n += 4) {
    const float w0 = __ldcs(W + (n + 0) * K + k);
    const float w1 = __ldcs(W + (n + 1) * K + k);
    const float w2 = __ldcs(W + (n + 2) * K + k);
    const float w3 = __ldcs(W + (n + 3) * K + k);
    acc0 += fabsf(w0) * __ldg(z + n + 0);
    acc1 += fabsf(w1) * __ldg(z + n + 1);
    acc2 += fabsf(w2) * __ldg(z + n + 2);
    acc3 += fabsf(w3) * __ldg(z + n + 3);
  }
  for (; n < n1; ++n) acc0 += fabsf(__ldcs(W + n * K + k)) * __ldg(z + n);
  part[s * K + k] = (acc0 + acc1) + (acc2 + acc3);
}

__device__ __forceinline__ double block_sum(double x, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = x;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
  return t;  // valid in thread 0
}

// y[k] = sum_s part[s][k] in a fixed order; accumulates ||y||^2.
__global__ void __launch_bounds__(256) svid_colsum_kernel(const float* __restrict__ part, int splits, int64_t K,
                                                          float* __restrict__ y, SvidScalars* sc) {
  if (svid_skip(sc, false, false)) return;
  __shared__ double red[8];
  double local = 0.0;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < K; k += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += part[(int64_t)s * K + k];
    y[k] = acc;
    local += (double)acc * (double)acc;
  }
  const double t = block_sum(local, red);
  if (threadIdx.x == 0) atomicAdd(&sc->yy, t);
}

// v <- y / ||y||; accumulates ||v_new - v||^2.  ||y|| == 0 leaves v unchanged.  The last
// block to finish takes the stopping decision and clears the accumulators for the next
// iteration (every block has read yy before it arrives).
__global__ void __launch_bounds__(256) svid_update_kernel(const float* __restrict__ y, float* __restrict__ v,
                                                          int64_t K, SvidScalars* sc, double tol2) {
  if (svid_skip(sc, false, false)) return;
  __shared__ double red[8];
  const double yy = *reinterpret_cast<const volatile double*>(&sc->yy);
  double local = 0.0;
  if (yy > 0.0) {
    const float inv = (float)(1.0 / sqrt(yy));
    for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < K;
         k += (int64_t)gridDim.x * blockDim.x) {
      const float nv = y[k] * inv;
      const double d = (double)nv - (double)v[k];
      local += d * d;
      v[k] = nv;
    }
  }
  const double t = block_sum(local, red);
  if (threadIdx.x == 0) {
    atomicAdd(&sc->diff2, t);
    __threadfence();
    if (atomicAdd(&sc->arrived, 1u) == gridDim.x - 1) {
      __threadfence();
      const double d2 = *reinterpret_cast<const volatile double*>(&sc->diff2);
      sc->iters += 1;
      if (isnan(yy) || isnan(d2))
        sc->state = kNan;
      else if (!(yy > 0.0) || d2 <= tol2)  // an all-zero |W| stops at once
        sc->state = kConverged;
      sc->yy = 0.0;
      sc->diff2 = 0.0;
      sc->arrived = 0u;
    }
  }
}

// a = z / sqrt(sigma1), b = sqrt(sigma1) v, sigma1 = ||z||.
__global__ void svid_finish_kernel(const float* __restrict__ z, const float* __restrict__ v, int64_t N, int64_t K,
                                   const SvidScalars* sc, float* a, float* b, float* sigma1, bool force) {
  if (svid_skip(sc, true, force)) return;
  const double s = sqrt(sc->zz);
  const bool zero = !(s > 0.0);
  const float ra = zero ? 0.f : (float)(1.0 / sqrt(s));
  const float rb = zero ? 0.f : (float)sqrt(s);
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t n = tid; n < N; n += stride) a[n] = z[n] * ra;
  for (int64_t k = tid; k < K; k += stride) b[k] = v[k] * rb;
  if (tid == 0 && sigma1) *sigma1 = (float)s;
}

}  // namespace

size_t svid_workspace_bytes(int64_t N, int64_t K) { return SvidLayout(N, K).total; }

ob_status run_svid(const float* W, int64_t N, int64_t K, float* a, float* b, float* sigma1, int max_iters,
                   float tol, int* iters_out, void* ws, const LaunchCtx& c) {
  const SvidLayout L(N, K);
  char* base = static_cast<char*>(ws);
  SvidScalars* sc = reinterpret_cast<SvidScalars*>(base);
  float* v = reinterpret_cast<float*>(base + L.off_v);
  float* z = reinterpret_cast<float*>(base + L.off_z);
  float* y = reinterpret_cast<float*>(base + L.off_y);
  float* part = reinterpret_cast<float*>(base + L.off_part);
  cudaStream_t st = c.stream;

  const int vec_blocks = (int)std::min<int64_t>((K + 255) / 256, (int64_t)c.num_sms * 4);
  const int row_blocks = (int)std::min<int64_t>((N + 7) / 8, (int64_t)c.num_sms * 16);
  const int64_t stripes = (K + kColThreads - 1) / kColThreads;
  int64_t splits = (4 * (int64_t)c.num_sms + stripes - 1) / stripes;
  splits = std::max<int64_t>(1, std::min<int64_t>(splits, std::min<int64_t>(kSplitsMax, N)));
  const int64_t rows_per_split = (N + splits - 1) / splits;
  splits = (N + rows_per_split - 1) / rows_per_split;

  if (cudaMemsetAsync(sc, 0, sizeof(SvidScalars), st) != cudaSuccess) return OB_ERR_CUDA;
  svid_init_kernel<<<vec_blocks, 256, 0, st>>>(v, K);
  if (cudaGetLastError() != cudaSuccess) return OB_ERR_CUDA;

  const double tol2 = (double)tol * (double)tol;
  int queued = 0;
  for (;;) {
    const int nb = std::min(kBatch, max_iters - queued);
    for (int i = 0; i < nb; ++i) {
      svid_rowdot_kernel<<<row_blocks, 256, 0, st>>>(W, N, K, v, z, sc, false, false);
      svid_coldot_kernel<<<dim3((unsigned)stripes, (unsigned)splits), kColThreads, 0, st>>>(W, N, K, z, part,
                                                                                          rows_per_split, sc);
      svid_colsum_kernel<<<vec_blocks, 256, 0, st>>>(part, (int)splits, K, y, sc);
      svid_update_kernel<<<vec_blocks, 256, 0, st>>>(y, v, K, sc, tol2);
    }
    queued += nb;
    const bool force = queued >= max_iters;  // the cap: finish with the last iterate
    svid_rowdot_kernel<<<row_blocks, 256, 0, st>>>(W, N, K, v, z, sc, true, force);
    svid_finish_kernel<<<vec_blocks, 256, 0, st>>>(z, v, N, K, sc, a, b, sigma1, force);
    if (cudaGetLastError() != cudaSuccess) return OB_ERR_CUDA;
    SvidScalars host;
    if (cudaMemcpyAsync(&host, sc, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess) return OB_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return OB_ERR_CUDA;
    if (iters_out) *iters_out = host.iters;
    if (host.state == kNan) return OB_ERR_NAN;
    if (host.state == kConverged || force) {
      if (std::isnan(host.zz)) return OB_ERR_NAN;
      return host.state == kConverged ? OB_OK : OB_ERR_NOT_CONVERGED;
    }
  }
}

}  // namespace ob
