// dbf_factorize.cu -- the DBF factorisation W -> (S_A, S_B, a, m, b) on the GPU.
//
// "Addition is almost all you need: Compressing large language models with double
// binary factorization" (gist.science), "Optimalisatie en Training": a heuristic of
// alternating minimisation with ADMM, the binary constraints met by an SVID-based
// projection.  The page gives no steps; the reading implemented here is the oracle's
// (oracle/dbf_factorize.py) with its sketch start:
//
//   start   A = W Ω;  B = argmin ||W - A B||^2 + eps ||B||^2, eps = 0.1 trace(A^T A) / r
//           (a ridge far above fp32 rounding of A^T A, so a rank-deficient W Ω stays
//           well posed);
//           Z_A, Z_B their SVID projections, scaled duals U_A = U_B = 0.
//   sweep   admm_iters ADMM steps on the left factor (Z_B fixed), then as many on the
//           right factor (Z_A fixed).  One step:
//             X <- the solution of X (G + rho I) = R,   G = F^T F,
//                  R = op(W) F + rho (Z - U),           rho = rho_rel trace(G) / r
//             Z <- SVID projection of X + U:  diag(u) Sign(X + U) diag(v), u v^T the
//                  rank-1 SVID of |X + U|
//             U <- U + X - Z
//           The right factor is kept transposed (K x r), so both steps have this form:
//           left op(W) = W, F = Z_B^T; right op(W) = W^T, F = Z_A.
//   keep    the best ||W - Z_A Z_B||_F over the start and the sweeps.
//   refit   with the signs fixed, a, then b, then m by exact least squares,
//           refit_rounds times.
//
// The r x r systems are solved by conjugate gradients over the rows of X (each row is
// one right-hand side of the symmetric positive definite G + rho I), warm-started from
// the previous X, a fixed number of iterations; the oracle solves exactly, so the two
// agree to the iteration's convergence.  The m refit's system is solved from zero to a
// relative residual of 1e-6.  Dense products run on a register-blocked fp32
// SIMT GEMM (offline work: a few hundred N x K x r products per weight matrix).
#include <algorithm>
#include <cmath>

#include "ob_device.cuh"
#include "ob_internal.h"

namespace ob {
namespace {

constexpr float kSketchRidge = 0.1f;  // the start's ridge, in units of trace(A^T A) / r

// ------------------------------------------------------------------ bounds
// Every device buffer below travels with its length in floats.  Before each launch the
// host checks that the highest element the launch can reach lies inside the buffer it
// was given; a failed check returns OB_ERR_DEVICE_BOUNDS and launches nothing.  Built
// with -DOB_DEBUG_BOUNDS (python -m binary_weight_gemm_b200.build --debug-bounds), the
// GEMM and conjugate-gradient kernels also check every index they form against those
// lengths on the device: an index outside records OB_DEVERR_BOUNDS in the device error
// word and the access is skipped.
struct Buf {
  float* p;
  int64_t n;  // length in floats
};

#ifdef OB_DEBUG_BOUNDS
__device__ __forceinline__ bool idx_ok(int64_t i, int64_t n, unsigned* err) {
  if (i >= 0 && i < n) return true;
  record_error(err, OB_DEVERR_BOUNDS);
  return false;
}
#else
__device__ __forceinline__ bool idx_ok(int64_t, int64_t, unsigned*) { return true; }
#endif

#define OB_NEED(cond)                              \
  do {                                             \
    if (!(cond)) return OB_ERR_DEVICE_BOUNDS;      \
  } while (0)

// ------------------------------------------------------------------ fp32 GEMM
// C (M x N, row stride ldc) = alpha * op(A) * op(B) + beta * C, all row-major.
// op(A) is M x K: A itself (M x K, stride lda) or, with TA, the transpose of A (K x M).
// op(B) is K x N: B itself (K x N, stride ldb) or, with TB, the transpose of B (N x K).
// 128 x 128 tiles, k steps of 8 through two shared-memory buffers (the next step's
// elements are loaded into registers while the current one is multiplied), 256 threads
// with 8 x 8 outputs each: rows ty*4 + i and 64 + ty*4 + i, columns tx*4 + j and
// 64 + tx*4 + j (i, j < 4), so every shared-memory read is a float4.  Rows of the tiles
// are padded to 132 floats: the stores of a warp then fall in 32 different banks.
// beta == 0 never reads C.  nA, nB, nC: the operands' lengths (device-side checks).
constexpr int kTile = 128;
constexpr int kKStep = 8;
constexpr int kPad = kTile + 4;

template <bool TA, bool TB>
__global__ void __launch_bounds__(256) sgemm_kernel(int64_t M, int64_t N, int64_t K, float alpha,
                                                    const float* __restrict__ A, int64_t lda, int64_t nA,
                                                    const float* __restrict__ B, int64_t ldb, int64_t nB,
                                                    float beta, float* __restrict__ C, int64_t ldc, int64_t nC,
                                                    unsigned* err) {
  __shared__ __align__(16) float As[2][kKStep][kPad];
  __shared__ __align__(16) float Bs[2][kKStep][kPad];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = (int64_t)blockIdx.y * kTile, n0 = (int64_t)blockIdx.x * kTile;
  // Element e = tid + 256 q of each 128 x 8 tile; consecutive threads walk the operand's
  // contiguous dimension.
  float ra[4], rb[4];
  auto load = [&](int64_t k0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + 256 * q;
      const int am = TA ? (e & 127) : (e >> 3), ak = TA ? (e >> 7) : (e & 7);
      const int64_t gm = m0 + am, gka = k0 + ak;
      const int64_t ia = TA ? gka * lda + gm : gm * lda + gka;
      ra[q] = (gm < M && gka < K && idx_ok(ia, nA, err)) ? A[ia] : 0.f;
      const int bn = TB ? (e >> 3) : (e & 127), bk = TB ? (e & 7) : (e >> 7);
      const int64_t gn = n0 + bn, gkb = k0 + bk;
      const int64_t ib = TB ? gn * ldb + gkb : gkb * ldb + gn;
      rb[q] = (gn < N && gkb < K && idx_ok(ib, nB, err)) ? B[ib] : 0.f;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + 256 * q;
      const int am = TA ? (e & 127) : (e >> 3), ak = TA ? (e >> 7) : (e & 7);
      As[buf][ak][am] = ra[q];
      const int bn = TB ? (e >> 3) : (e & 127), bk = TB ? (e & 7) : (e >> 7);
      Bs[buf][bk][bn] = rb[q];
    }
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  load(0);
  store(0);
  __syncthreads();
  int buf = 0;
  for (int64_t k0 = 0; k0 < K; k0 += kKStep) {
    const bool more = k0 + kKStep < K;
    if (more) load(k0 + kKStep);
#pragma unroll
    for (int kk = 0; kk < kKStep; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    // The other buffer was last read in the previous step, which every thread finished
    // before that step's barrier.
    if (more) store(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn >= N) continue;
      const int64_t ic = gm * ldc + gn;
      if (!idx_ok(ic, nC, err)) continue;
      float* c = C + ic;
      *c = beta == 0.f ? alpha * acc[i][j] : fmaf(alpha, acc[i][j], beta * *c);
    }
  }
}

ob_status gemm(bool ta, bool tb, int64_t M, int64_t N, int64_t K, float alpha, Buf A, int64_t lda, Buf B,
               int64_t ldb, float beta, Buf C, int64_t ldc, const LaunchCtx& lc) {
  if (M == 0 || N == 0) return OB_OK;
  // Leading dimensions cover a row, and the highest element of each operand is inside it.
  OB_NEED(lda >= (ta ? M : K) && ldb >= (tb ? K : N) && ldc >= N);
  if (K > 0) {
    OB_NEED((ta ? (K - 1) * lda + M : (M - 1) * lda + K) <= A.n);
    OB_NEED((tb ? (N - 1) * ldb + K : (K - 1) * ldb + N) <= B.n);
  }
  OB_NEED((M - 1) * ldc + N <= C.n);
  const dim3 grid((unsigned)((N + kTile - 1) / kTile), (unsigned)((M + kTile - 1) / kTile));
  if (grid.y > 65535u) return OB_ERR_UNSUPPORTED;
  const cudaStream_t s = lc.stream;
  if (!ta && !tb)
    sgemm_kernel<false, false><<<grid, 256, 0, s>>>(M, N, K, alpha, A.p, lda, A.n, B.p, ldb, B.n, beta, C.p,
                                                     ldc, C.n, lc.err);
  else if (ta && !tb)
    sgemm_kernel<true, false><<<grid, 256, 0, s>>>(M, N, K, alpha, A.p, lda, A.n, B.p, ldb, B.n, beta, C.p,
                                                    ldc, C.n, lc.err);
  else if (!ta && tb)
    sgemm_kernel<false, true><<<grid, 256, 0, s>>>(M, N, K, alpha, A.p, lda, A.n, B.p, ldb, B.n, beta, C.p,
                                                    ldc, C.n, lc.err);
  else
    sgemm_kernel<true, true><<<grid, 256, 0, s>>>(M, N, K, alpha, A.p, lda, A.n, B.p, ldb, B.n, beta, C.p,
                                                   ldc, C.n, lc.err);
  return cudaGetLastError() == cudaSuccess ? OB_OK : OB_ERR_CUDA;
}

// ------------------------------------------------------------------ elementwise

unsigned blocks_for(int64_t n) {
  const int64_t b = (n + 255) / 256;
  return (unsigned)(b < 4096 ? (b < 1 ? 1 : b) : 4096);
}

#define OB_GRID_STRIDE(i, n) \
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (n); i += (int64_t)gridDim.x * blockDim.x)

// Z = diag(u) Sign(M) diag(v) (rows x cols); Sign(x) = -1 iff x < 0.
__global__ void structured_kernel(const float* __restrict__ M, const float* __restrict__ u,
                                  const float* __restrict__ v, float* __restrict__ Z, int64_t rows, int64_t cols) {
  OB_GRID_STRIDE(i, rows * cols) {
    const int64_t r = i / cols, c = i - r * cols;
    const float s = M[i] < 0.f ? -1.f : 1.f;
    Z[i] = s * u[r] * v[c];
  }
}

// R += rho (Z - U)
__global__ void admm_rhs_kernel(float* __restrict__ R, const float* __restrict__ Z, const float* __restrict__ U,
                                const float* __restrict__ rho_p, int64_t n) {
  const float rho = *rho_p;
  OB_GRID_STRIDE(i, n) R[i] += rho * (Z[i] - U[i]);
}

// out = x + y
__global__ void add_kernel(const float* __restrict__ x, const float* __restrict__ y, float* __restrict__ out,
                           int64_t n) {
  OB_GRID_STRIDE(i, n) out[i] = x[i] + y[i];
}

// U += X - Z
__global__ void dual_kernel(float* __restrict__ U, const float* __restrict__ X, const float* __restrict__ Z,
                            int64_t n) {
  OB_GRID_STRIDE(i, n) U[i] += X[i] - Z[i];
}

// out = x * y (elementwise; out may be x)
__global__ void mul_kernel(const float* x, const float* y, float* out, int64_t n) {
  OB_GRID_STRIDE(i, n) out[i] = x[i] * y[i];
}

__global__ void fill_kernel(float* __restrict__ x, float v, int64_t n) {
  OB_GRID_STRIDE(i, n) x[i] = v;
}

// out (cols x rows) = in (rows x cols)^T
__global__ void transpose_kernel(const float* __restrict__ in, float* __restrict__ out, int64_t rows,
                                 int64_t cols) {
  OB_GRID_STRIDE(i, rows * cols) {
    const int64_t r = i / cols, c = i - r * cols;
    out[c * rows + r] = in[i];
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// *out = scale * trace(G) / r (G r x r), clamped at 0.  One block of 256 threads.
__global__ void trace_scale_kernel(const float* __restrict__ G, int64_t r, float scale, float* __restrict__ out) {
  __shared__ double part[256];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < r; i += 256) s += (double)G[i * r + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double v = (double)scale * part[0] / (double)r;
    *out = v > 0.0 ? (float)v : 0.f;
  }
}

// *acc += sum_i (W[i] - C[i])^2 (double, one atomic per block).
__global__ void sqdiff_kernel(const float* __restrict__ W, const float* __restrict__ C, int64_t n,
                              double* __restrict__ acc) {
  __shared__ double part[256];
  double s = 0.0;
  OB_GRID_STRIDE(i, n) {
    const double d = (double)W[i] - (double)C[i];
    s += d * d;
  }
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) atomicAdd(acc, part[0]);
}

// Per row n (one warp): out[n] = <W_n, C_n> / ||C_n||^2, 0 where ||C_n|| = 0.
__global__ void row_ratio_kernel(const float* __restrict__ W, const float* __restrict__ C, int64_t rows,
                                 int64_t cols, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  float num = 0.f, den = 0.f;
  for (int64_t j = lane; j < cols; j += 32) {
    const float c = C[row * cols + j];
    num = fmaf(W[row * cols + j], c, num);
    den = fmaf(c, c, den);
  }
  num = warp_sum(num);
  den = warp_sum(den);
  if (lane == 0) out[row] = den > 0.f ? num / den : 0.f;
}

// Per column k (one thread): ratio: out[k] = <X[:, k], Y[:, k]> / ||Y[:, k]||^2 (0 where
// the norm is 0); otherwise out[k] = <X[:, k], Y[:, k]>.
__global__ void col_dot_kernel(const float* __restrict__ X, const float* __restrict__ Y, int64_t rows,
                               int64_t cols, bool ratio, float* __restrict__ out) {
  OB_GRID_STRIDE(k, cols) {
    double num = 0.0, den = 0.0;
    for (int64_t i = 0; i < rows; ++i) {
      const double y = Y[i * cols + k];
      num += (double)X[i * cols + k] * y;
      den += y * y;
    }
    out[k] = ratio ? (den > 0.0 ? (float)(num / den) : 0.f) : (float)num;
  }
}

// q = G x for the symmetric r x r matrix G (one warp per row of G): the one-row case of
// the conjugate-gradient product x G.
__global__ void symv_kernel(const float* __restrict__ G, const float* __restrict__ x, float* __restrict__ q,
                            int64_t r, int64_t nG, unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= r) return;
  float s = 0.f;
  for (int64_t j = lane; j < r; j += 32) {
    const int64_t i = row * r + j;
    if (idx_ok(i, nG, err)) s = fmaf(G[i], x[j], s);
  }
  s = warp_sum(s);
  if (lane == 0) q[row] = s;
}

// Conjugate gradients on X (G + rho I) = R, row by row (one warp per row); every
// rows x r operand holds n >= rows * r floats.
// Start: T = X G (given); Res = R - T - rho X (in place of R), P = Res,
// rr = rr_start = ||Res_n||^2.
__global__ void cg_init_kernel(const float* __restrict__ X, float* __restrict__ R, const float* __restrict__ T,
                               float* __restrict__ P, float* __restrict__ rr, float* __restrict__ rr_start,
                               const float* __restrict__ rho_p, int64_t rows, int64_t r, int64_t n,
                               unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float rho = *rho_p;
  float s = 0.f;
  for (int64_t j = lane; j < r; j += 32) {
    const int64_t i = row * r + j;
    if (!idx_ok(i, n, err)) continue;
    const float res = R[i] - T[i] - rho * X[i];
    R[i] = res;
    P[i] = res;
    s = fmaf(res, res, s);
  }
  s = warp_sum(s);
  if (lane == 0) {
    rr[row] = s;
    rr_start[row] = s;
  }
}

// One iteration, given Q = P G: alpha = rr / <P, Q + rho P>; X += alpha P;
// Res -= alpha (Q + rho P); beta = ||Res||^2 / rr; P = Res + beta P.  A row stops moving
// once ||Res||^2 <= tol2 * rr_start (its relative residual reached sqrt(tol2)), or when
// its curvature is not positive or its residual is zero.
__global__ void cg_step_kernel(float* __restrict__ X, float* __restrict__ Res, float* __restrict__ P,
                               const float* __restrict__ Q, float* __restrict__ rr,
                               const float* __restrict__ rr_start, const float* __restrict__ rho_p, float tol2,
                               int64_t rows, int64_t r, int64_t n, unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float rho = *rho_p;
  const int64_t base = row * r;
  float pq = 0.f;
  for (int64_t j = lane; j < r; j += 32)
    if (idx_ok(base + j, n, err)) pq = fmaf(P[base + j], Q[base + j] + rho * P[base + j], pq);
  pq = warp_sum(pq);
  const float rr0 = rr[row];
  const bool live = rr0 > 0.f && rr0 > tol2 * rr_start[row];
  const float alpha = (live && pq > 0.f && isfinite(pq)) ? rr0 / pq : 0.f;
  float rn = 0.f;
  for (int64_t j = lane; j < r; j += 32) {
    const int64_t i = base + j;
    if (!idx_ok(i, n, err)) continue;
    const float pj = P[i];
    X[i] = fmaf(alpha, pj, X[i]);
    const float nr = Res[i] - alpha * (Q[i] + rho * pj);
    Res[i] = nr;
    rn = fmaf(nr, nr, rn);
  }
  rn = warp_sum(rn);
  const float beta = (alpha != 0.f && rr0 > 0.f) ? rn / rr0 : 0.f;
  for (int64_t j = lane; j < r; j += 32)
    if (idx_ok(base + j, n, err)) P[base + j] = Res[base + j] + beta * P[base + j];
  if (lane == 0) rr[row] = alpha != 0.f ? rn : 0.f;
}

// ------------------------------------------------------------------ workspace

size_t al(size_t x) { return (x + 255) & ~size_t(255); }

struct FactLayout {
  size_t XA, ZA, UA, MA, MAb, XB, ZB, UB, MB, MBb, R, P, Q, G, G2, C;
  size_t uA, vA, uAb, vAb, uB, vB, uBb, vBb, ones, rr, rr0, h, rho, zero, acc, svid, total;
  FactLayout(int64_t N, int64_t K, int64_t r) {
    const size_t f = sizeof(float);
    const size_t L = (size_t)(N > K ? N : K);
    const size_t V = (size_t)(L > (size_t)r ? L : (size_t)r);
    size_t o = 0;
    auto take = [&o](size_t bytes) {
      const size_t at = o;
      o = al(o + bytes);
      return at;
    };
    XA = take(f * N * r); ZA = take(f * N * r); UA = take(f * N * r); MA = take(f * N * r); MAb = take(f * N * r);
    XB = take(f * K * r); ZB = take(f * K * r); UB = take(f * K * r); MB = take(f * K * r); MBb = take(f * K * r);
    R = take(f * L * r); P = take(f * L * r); Q = take(f * L * r);
    G = take(f * r * r); G2 = take(f * r * r);
    C = take(f * N * K);
    uA = take(f * N); vA = take(f * r); uAb = take(f * N); vAb = take(f * r);
    uB = take(f * K); vB = take(f * r); uBb = take(f * K); vBb = take(f * r);
    ones = take(f * V); rr = take(f * L); rr0 = take(f * L); h = take(f * r);
    rho = take(f); zero = take(f); acc = take(sizeof(double));
    svid = take(svid_workspace_bytes((int64_t)L, r));
    total = o;
  }
};

#define OB_TRY_CUDA(x)                      \
  do {                                      \
    if ((x) != cudaSuccess) return OB_ERR_CUDA; \
  } while (0)
#define OB_TRY(x)                \
  do {                           \
    const ob_status st_ = (x);   \
    if (st_ != OB_OK) return st_; \
  } while (0)

ob_status launched() { return cudaGetLastError() == cudaSuccess ? OB_OK : OB_ERR_CUDA; }

// X (rows x r) <- CG solution of X (G + rho I) = R, warm-started from X, at most `iters`
// iterations; a row stops once its relative residual reaches sqrt(tol2) (tol2 = 0: never
// early).  R is overwritten (the residual); P, Q (rows x r) and rr, rr0 (rows) are scratch.
ob_status cg_solve(Buf X, Buf R, Buf G, const float* rho, int64_t rows, int64_t r, int iters, float tol2, Buf P,
                   Buf Q, Buf rr, Buf rr0, const LaunchCtx& lc) {
  const int64_t n = rows * r;
  OB_NEED(X.n >= n && R.n >= n && P.n >= n && Q.n >= n && rr.n >= rows && rr0.n >= rows && G.n >= r * r);
  const cudaStream_t s = lc.stream;
  const unsigned rb = (unsigned)((rows + 7) / 8);  // 8 warps per block, one row each
  const unsigned gb = (unsigned)((r + 7) / 8);
  auto times_g = [&](Buf in) -> ob_status {  // Q = in G
    if (rows == 1) {
      symv_kernel<<<gb, 256, 0, s>>>(G.p, in.p, Q.p, r, G.n, lc.err);
      return launched();
    }
    return gemm(false, false, rows, r, r, 1.f, in, r, G, r, 0.f, Q, r, lc);
  };
  OB_TRY(times_g(X));
  cg_init_kernel<<<rb, 256, 0, s>>>(X.p, R.p, Q.p, P.p, rr.p, rr0.p, rho, rows, r, n, lc.err);
  OB_TRY(launched());
  for (int t = 0; t < iters; ++t) {
    OB_TRY(times_g(P));
    cg_step_kernel<<<rb, 256, 0, s>>>(X.p, R.p, P.p, Q.p, rr.p, rr0.p, rho, tol2, rows, r, n, lc.err);
    OB_TRY(launched());
  }
  return OB_OK;
}

// Z = diag(u) Sign(M) diag(v) with (u, v) the rank-1 SVID of |M| (rows x r).  A power
// iteration that reaches its cap keeps its last iterate, as the SVID entry point does.
ob_status project(Buf M, int64_t rows, int64_t r, Buf u, Buf v, Buf Z, void* svid_ws, const LaunchCtx& lc) {
  OB_NEED(M.n >= rows * r && Z.n >= rows * r && u.n >= rows && v.n >= r);
  const ob_status st = run_svid(M.p, rows, r, u.p, v.p, nullptr, 200, 1e-6f, nullptr, svid_ws, lc);
  if (st != OB_OK && st != OB_ERR_NOT_CONVERGED) return st;
  structured_kernel<<<blocks_for(rows * r), 256, 0, lc.stream>>>(M.p, u.p, v.p, Z.p, rows, r);
  return launched();
}

// Z = diag(u) Sign(M) diag(v), M rows x cols.
ob_status structured(Buf M, Buf u, Buf v, Buf Z, int64_t rows, int64_t cols, cudaStream_t s) {
  OB_NEED(M.n >= rows * cols && Z.n >= rows * cols && u.n >= rows && v.n >= cols);
  structured_kernel<<<blocks_for(rows * cols), 256, 0, s>>>(M.p, u.p, v.p, Z.p, rows, cols);
  return launched();
}

// ||W - Z_A Z_Bt^T||_F (host value; synchronises).  C: N x K scratch.
ob_status frob_error(Buf W, Buf ZA, Buf ZBt, int64_t N, int64_t K, int64_t r, Buf C, double* acc,
                     const LaunchCtx& lc, double* out) {
  const cudaStream_t s = lc.stream;
  OB_TRY(gemm(false, true, N, K, r, 1.f, ZA, r, ZBt, r, 0.f, C, K, lc));
  OB_NEED(W.n >= N * K && C.n >= N * K);
  OB_TRY_CUDA(cudaMemsetAsync(acc, 0, sizeof(double), s));
  sqdiff_kernel<<<blocks_for(N * K), 256, 0, s>>>(W.p, C.p, N * K, acc);
  OB_TRY(launched());
  double h = 0.0;
  OB_TRY_CUDA(cudaMemcpyAsync(&h, acc, sizeof(double), cudaMemcpyDeviceToHost, s));
  OB_TRY_CUDA(cudaStreamSynchronize(s));
  if (!std::isfinite(h)) return OB_ERR_NAN;
  *out = std::sqrt(h);
  return OB_OK;
}

// dst[0, n) = src[0, n) (device to device, stream-ordered).
ob_status copy(Buf dst, Buf src, int64_t n, cudaStream_t s) {
  OB_NEED(dst.n >= n && src.n >= n);
  OB_TRY_CUDA(cudaMemcpyAsync(dst.p, src.p, sizeof(float) * (size_t)n, cudaMemcpyDeviceToDevice, s));
  return OB_OK;
}

ob_status zero(Buf dst, int64_t n, cudaStream_t s) {
  OB_NEED(dst.n >= n);
  OB_TRY_CUDA(cudaMemsetAsync(dst.p, 0, sizeof(float) * (size_t)n, s));
  return OB_OK;
}

}  // namespace

size_t dbf_factorize_workspace_bytes(int64_t N, int64_t K, int64_t r) { return FactLayout(N, K, r).total; }

ob_status run_dbf_factorize(const float* W_in, int64_t N, int64_t K, int64_t r, const float* omega_in,
                            int sweeps, int admm_iters, int cg_iters, float rho_rel, int refit_rounds,
                            uint32_t* SA_packed, uint32_t* SB_packed, float* a_out, float* m_out, float* b_out,
                            float* history, float* best_out, float* error_out, void* workspace,
                            const LaunchCtx& lc) {
  const FactLayout Lo(N, K, r);
  const int64_t L = std::max<int64_t>(N, K);
  const int64_t V = std::max<int64_t>(L, r);
  char* base = static_cast<char*>(workspace);
  auto F = [base](size_t off, int64_t n) { return Buf{reinterpret_cast<float*>(base + off), n}; };
  const Buf XA = F(Lo.XA, N * r), ZA = F(Lo.ZA, N * r), UA = F(Lo.UA, N * r), MA = F(Lo.MA, N * r),
            MAb = F(Lo.MAb, N * r);
  const Buf XB = F(Lo.XB, K * r), ZB = F(Lo.ZB, K * r), UB = F(Lo.UB, K * r), MB = F(Lo.MB, K * r),
            MBb = F(Lo.MBb, K * r);
  const Buf R = F(Lo.R, L * r), P = F(Lo.P, L * r), Q = F(Lo.Q, L * r), G = F(Lo.G, r * r),
            G2 = F(Lo.G2, r * r), C = F(Lo.C, N * K);
  const Buf uA = F(Lo.uA, N), vA = F(Lo.vA, r), uAb = F(Lo.uAb, N), vAb = F(Lo.vAb, r);
  const Buf uB = F(Lo.uB, K), vB = F(Lo.vB, r), uBb = F(Lo.uBb, K), vBb = F(Lo.vBb, r);
  const Buf ones = F(Lo.ones, V), rr = F(Lo.rr, L), rr0 = F(Lo.rr0, L), h = F(Lo.h, r);
  float* rho = F(Lo.rho, 1).p;
  float* zero_p = F(Lo.zero, 1).p;
  double* acc = reinterpret_cast<double*>(base + Lo.acc);
  void* svid_ws = base + Lo.svid;
  // The caller's buffers (their lengths are the documented shapes).
  const Buf W{const_cast<float*>(W_in), N * K}, omega{const_cast<float*>(omega_in), K * r};
  const Buf a{a_out, N}, m{m_out, r}, b{b_out, K};
  const cudaStream_t s = lc.stream;

  fill_kernel<<<blocks_for(V), 256, 0, s>>>(ones.p, 1.f, V);
  fill_kernel<<<1, 32, 0, s>>>(zero_p, 0.f, 1);
  OB_TRY(launched());

  // ---- start: A = W Ω; B^T (K x r) solves B^T (A^T A + eps I) = W^T A.
  OB_TRY(gemm(false, false, N, r, K, 1.f, W, K, omega, r, 0.f, XA, r, lc));
  OB_TRY(gemm(true, false, r, r, N, 1.f, XA, r, XA, r, 0.f, G, r, lc));
  trace_scale_kernel<<<1, 256, 0, s>>>(G.p, r, kSketchRidge, rho);
  OB_TRY(launched());
  OB_TRY(gemm(true, false, K, r, N, 1.f, W, K, XA, r, 0.f, R, r, lc));
  OB_TRY(zero(XB, K * r, s));
  OB_TRY(cg_solve(XB, R, G, rho, K, r, 4 * cg_iters, 0.f, P, Q, rr, rr0, lc));
  OB_TRY(copy(MA, XA, N * r, s));
  OB_TRY(copy(MB, XB, K * r, s));
  OB_TRY(project(MA, N, r, uA, vA, ZA, svid_ws, lc));
  OB_TRY(project(MB, K, r, uB, vB, ZB, svid_ws, lc));
  OB_TRY(zero(UA, N * r, s));
  OB_TRY(zero(UB, K * r, s));

  auto keep_best = [&]() -> ob_status {
    OB_TRY(copy(MAb, MA, N * r, s));
    OB_TRY(copy(MBb, MB, K * r, s));
    OB_TRY(copy(uAb, uA, N, s));
    OB_TRY(copy(vAb, vA, r, s));
    OB_TRY(copy(uBb, uB, K, s));
    OB_TRY(copy(vBb, vB, r, s));
    return OB_OK;
  };
  double best = 0.0;
  OB_TRY(frob_error(W, ZA, ZB, N, K, r, C, acc, lc, &best));
  OB_TRY(keep_best());

  // ---- sweeps.  step(): one ADMM step on the factor X (rows x r) with the other factor F
  // (frows x r) fixed; op(W) F is W F (left: F = Z_B^T, K x r) or W^T F (right: F = Z_A).
  auto step = [&](bool left, Buf X, Buf Z, Buf U, Buf Mx, Buf u, Buf v, Buf Fo, int64_t rows,
                  int64_t frows) -> ob_status {
    const int64_t n = rows * r;
    OB_NEED(X.n >= n && Z.n >= n && U.n >= n && Mx.n >= n && R.n >= n);
    OB_TRY(gemm(true, false, r, r, frows, 1.f, Fo, r, Fo, r, 0.f, G, r, lc));
    trace_scale_kernel<<<1, 256, 0, s>>>(G.p, r, rho_rel, rho);
    OB_TRY(launched());
    if (left)
      OB_TRY(gemm(false, false, N, r, K, 1.f, W, K, Fo, r, 0.f, R, r, lc));
    else
      OB_TRY(gemm(true, false, K, r, N, 1.f, W, K, Fo, r, 0.f, R, r, lc));
    admm_rhs_kernel<<<blocks_for(n), 256, 0, s>>>(R.p, Z.p, U.p, rho, n);
    OB_TRY(launched());
    OB_TRY(cg_solve(X, R, G, rho, rows, r, cg_iters, 0.f, P, Q, rr, rr0, lc));
    add_kernel<<<blocks_for(n), 256, 0, s>>>(X.p, U.p, Mx.p, n);
    OB_TRY(launched());
    OB_TRY(project(Mx, rows, r, u, v, Z, svid_ws, lc));
    dual_kernel<<<blocks_for(n), 256, 0, s>>>(U.p, X.p, Z.p, n);
    return launched();
  };
  for (int sw = 0; sw < sweeps; ++sw) {
    for (int t = 0; t < admm_iters; ++t) OB_TRY(step(true, XA, ZA, UA, MA, uA, vA, ZB, N, K));
    for (int t = 0; t < admm_iters; ++t) OB_TRY(step(false, XB, ZB, UB, MB, uB, vB, ZA, K, N));
    double e = 0.0;
    OB_TRY(frob_error(W, ZA, ZB, N, K, r, C, acc, lc, &e));
    if (history) history[sw] = (float)e;
    if (e < best) {
      best = e;
      OB_TRY(keep_best());
    }
  }
  if (best_out) *best_out = (float)best;

  // ---- the kept iterate: a = u_A, m = v_A ⊙ v_B (v_B is Z_B's row scale: Z_B^T = diag(u_B) S_B^T diag(v_B)),
  // b = u_B; then the least-squares refits.  Dense forms built from the kept signs:
  //   Lm = S_A diag(m), Rb = (S_B diag(b))^T = diag(b) S_B^T, La = diag(a) S_A diag(m), Sb = S_B^T.
  OB_TRY(copy(a, uAb, N, s));
  OB_TRY(copy(b, uBb, K, s));
  mul_kernel<<<blocks_for(r), 256, 0, s>>>(vAb.p, vBb.p, m.p, r);
  OB_TRY(launched());
  const Buf Lx = XA;  // N x r scratch (the iterates are no longer needed)
  const Buf Rx = XB;  // K x r scratch
  // The m refit runs CG from zero to a relative residual of 1e-6 (at most max(4 cg_iters, r)
  // iterations): from zero, CG stays in the range of the matrix, so on a singular system it
  // tends to the least-squares solution of smallest norm, the one the oracle's lstsq returns.
  const int m_iters = (int)std::max<int64_t>(4 * (int64_t)cg_iters, r);
  for (int t = 0; t < refit_rounds; ++t) {
    // a: rows of R = Lm Rb^T against W.
    OB_TRY(structured(MAb, ones, m, Lx, N, r, s));
    OB_TRY(structured(MBb, b, ones, Rx, K, r, s));
    OB_TRY(gemm(false, true, N, K, r, 1.f, Lx, r, Rx, r, 0.f, C, K, lc));
    row_ratio_kernel<<<(unsigned)((N + 7) / 8), 256, 0, s>>>(W.p, C.p, N, K, a.p);
    OB_TRY(launched());
    // b: columns of C = La Sb^T against W.
    OB_TRY(structured(MAb, a, m, Lx, N, r, s));
    OB_TRY(structured(MBb, ones, ones, Rx, K, r, s));
    OB_TRY(gemm(false, true, N, K, r, 1.f, Lx, r, Rx, r, 0.f, C, K, lc));
    col_dot_kernel<<<blocks_for(K), 256, 0, s>>>(W.p, C.p, N, K, true, b.p);
    OB_TRY(launched());
    // m: (P^T P ∘ Q Q^T) m = h, P = diag(a) S_A (N x r), Qt = (S_B diag(b))^T (K x r),
    // h_j = sum_k (W^T P)[k, j] Qt[k, j].
    OB_TRY(structured(MAb, a, ones, Lx, N, r, s));
    OB_TRY(structured(MBb, b, ones, Rx, K, r, s));
    OB_TRY(gemm(true, false, r, r, N, 1.f, Lx, r, Lx, r, 0.f, G, r, lc));
    OB_TRY(gemm(true, false, r, r, K, 1.f, Rx, r, Rx, r, 0.f, G2, r, lc));
    mul_kernel<<<blocks_for(r * r), 256, 0, s>>>(G.p, G2.p, G.p, r * r);
    OB_TRY(launched());
    OB_TRY(gemm(true, false, K, r, N, 1.f, W, K, Lx, r, 0.f, R, r, lc));
    OB_NEED(R.n >= K * r && Rx.n >= K * r);
    col_dot_kernel<<<blocks_for(r), 256, 0, s>>>(R.p, Rx.p, K, r, false, h.p);
    OB_TRY(launched());
    OB_TRY(zero(m, r, s));
    OB_TRY(cg_solve(m, h, G, zero_p, 1, r, m_iters, 1e-12f, P, Q, rr, rr0, lc));
  }
  // Final error with the refitted scales: W_hat = La Rb^T.
  OB_TRY(structured(MAb, a, m, Lx, N, r, s));
  OB_TRY(structured(MBb, b, ones, Rx, K, r, s));
  double e = 0.0;
  OB_TRY(frob_error(W, Lx, Rx, N, K, r, C, acc, lc, &e));
  if (error_out) *error_out = (float)e;

  // ---- packed signs: S_A from the kept M_A (N x r); S_B from the kept M_B^T transposed.
  OB_TRY_CUDA(launch_pack_signs(MAb.p, N, r, SA_packed, lc));
  OB_NEED(R.n >= K * r);
  transpose_kernel<<<blocks_for(K * r), 256, 0, s>>>(MBb.p, R.p, K, r);  // R: r x K
  OB_TRY(launched());
  OB_TRY_CUDA(launch_pack_signs(R.p, r, K, SB_packed, lc));
  OB_TRY_CUDA(cudaStreamSynchronize(s));
  return OB_OK;
}

}  // namespace ob
