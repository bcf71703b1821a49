// api.cu -- the C ABI of libobgemm (declarations and contracts in include/obgemm.h).
//
// Host-side argument checks, kernel dispatch and the per-device error word.
// Checks run before any CUDA call, so a rejected call launches nothing.
#include <cstring>
#include <mutex>
#include <vector>

#include "ob_device.cuh"
#include "ob_internal.h"

// Device error word: bits OB_DEVERR_* set by kernels, read and cleared by ob_last_device_error.
__device__ unsigned g_ob_error_word;

// Static scratch for dbf_linear_noalloc: holds the DBF intermediate for callers
// that cannot allocate.  Reserved on every device that loads the library.
static __device__ __align__(256) unsigned char g_dbf_noalloc_scratch[OB_DBF_NOALLOC_SCRATCH_BYTES];

namespace ob {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  unsigned* err = nullptr;
  int num_sms = 0;
  int major = 0;
  bool ready = false;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

// Error word address, SM count and architecture of the current device (cached per device).
ob_status current_device(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OB_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ob_error_word) != cudaSuccess) return OB_ERR_CUDA;
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return OB_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return OB_ERR_CUDA;
    d.err = static_cast<unsigned*>(p);
    d.num_sms = sms;
    d.major = major;
    d.ready = true;
  }
  *out = d;
  return OB_OK;
}

ob_status make_ctx(void* stream, LaunchCtx* c) {
  DeviceInfo d;
  ob_status st = current_device(&d);
  if (st != OB_OK) return st;
  if (d.major != 10) return OB_ERR_UNSUPPORTED;  // sm_100 family only
  c->stream = static_cast<cudaStream_t>(stream);
  c->err = d.err;
  c->num_sms = d.num_sms;
  c->pdl = true;
  c->l2_prefetch = true;
  return OB_OK;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

ob_status zero_output(void* Y, int64_t M, int64_t N, int y_dtype, cudaStream_t s) {
  const size_t bytes = (size_t)M * (size_t)N * (y_dtype == OB_OUT_F32 ? 4 : 2);
  return cudaMemsetAsync(Y, 0, bytes, s) == cudaSuccess ? OB_OK : OB_ERR_CUDA;
}

ob_status status_of(cudaError_t e) {
  if (e == cudaSuccess) return OB_OK;
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) return OB_ERR_UNSUPPORTED;
  return OB_ERR_CUDA;
}

ob_status run_sign_gemm(const SignGemmArgs& g_in, int path, const LaunchCtx& c) {
  SignGemmArgs g = g_in;
  g.l2_prefetch = (c.pdl && c.l2_prefetch) ? 1 : 0;
  // Measured on B200 (4096 x 4096 layer, one call per CUDA-graph node): one token is
  // fastest on the table-driven CUDA-core kernel, 2..16 tokens on the warp-level
  // MMA kernel, more on the tcgen05 GEMM.  K beyond the tcgen05 GEMM's limit goes
  // to the warp-level MMA kernel, 16 tokens per launch.
  if (path == OB_PATH_AUTO) {
    path = g.M == 1 ? OB_PATH_SIMT : (g.M <= kDecodeMaxM ? OB_PATH_MMA_DECODE : OB_PATH_TC);
    if (path == OB_PATH_TC && g.K > sign_gemm_tc_max_k()) path = OB_PATH_MMA_DECODE;
  }
  cudaError_t e;
  switch (path) {
    case OB_PATH_SIMT: e = launch_sign_gemm_simt(g, c); break;
    case OB_PATH_MMA_DECODE: e = launch_sign_gemm_mma_decode(g, c); break;
    case OB_PATH_I8: e = launch_sign_gemm_i8(g, c); break;
    case OB_PATH_TC:
      // The CTA-pair kernel where it applies (bf16 Y, M >= 512, R >= 256, K <= 16384):
      // 1260 vs 1170 TFLOP/s for the one-CTA kernel at the prefill workload on B200.
      e = sign_gemm_tc2_supported(g) ? launch_sign_gemm_tc2(g, c) : launch_sign_gemm_tc(g, c);
      break;
    case OB_PATH_TC1: e = launch_sign_gemm_tc(g, c); break;
    default: return OB_ERR_UNSUPPORTED;
  }
  return status_of(e);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Largest M the int8 form of the layer stack takes (its activation limbs for up to two
// tokens fill one n8 tile).
constexpr int64_t kStackI8MaxM = 2;

// Largest N, K or r of dbf_factorize: its GEMM grid has one row of CTAs per 128 rows, so
// 2^22 rows keep grid.y at 32768, inside the 65535 limit.
constexpr int64_t kFactorizeMaxDim = (int64_t)1 << 22;

// Largest element count of any one matrix a call may describe (2^48, far past device
// memory): shapes are checked against it by division before any product of sizes is
// formed, so no size computation below can wrap.
constexpr int64_t kMaxElems = (int64_t)1 << 48;
bool elems_ok(int64_t rows, int64_t cols) { return rows == 0 || cols <= kMaxElems / rows; }

int sms_for_sizing() {
  DeviceInfo d;
  return current_device(&d) == OB_OK && d.num_sms > 0 ? d.num_sms : 148;  // B200 when no device
}

// K slices for a problem that runs on the one-CTA tcgen05 GEMM with few output tiles (1: no
// split).  The slices' partial sums are summed by a kernel that writes 4 outputs at a time,
// so N must be a multiple of 4.
int linear_split_k(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= kDecodeMaxM || N % 4 != 0 || K > sign_gemm_tc_max_k()) return 1;
  return tc_split_k(M, N, K, num_sms);
}

}  // namespace
}  // namespace ob

using namespace ob;

extern "C" {

const char* ob_status_string(int status) {
  switch (status) {
    case OB_OK: return "OB_OK";
    case OB_ERR_NULL: return "OB_ERR_NULL: a required pointer is NULL";
    case OB_ERR_SHAPE: return "OB_ERR_SHAPE: negative size, or K / r not a multiple of 32";
    case OB_ERR_ALIGN: return "OB_ERR_ALIGN: a pointer is not 16-byte aligned";
    case OB_ERR_NAN: return "OB_ERR_NAN: NaN in an input that must be finite";
    case OB_ERR_NOT_CONVERGED: return "OB_ERR_NOT_CONVERGED: SVID reached max_iters";
    case OB_ERR_WORKSPACE: return "OB_ERR_WORKSPACE: workspace missing or too small";
    case OB_ERR_CUDA: return "OB_ERR_CUDA: CUDA runtime error";
    case OB_ERR_DEVICE_TIMEOUT: return "OB_ERR_DEVICE_TIMEOUT: a bounded wait in a kernel ran out";
    case OB_ERR_UNSUPPORTED: return "OB_ERR_UNSUPPORTED: unsupported device, size or option";
    case OB_ERR_DEVICE_BOUNDS: return "OB_ERR_DEVICE_BOUNDS: a kernel refused an out-of-bounds access";
    default: return "unknown ob_status";
  }
}

int ob_version(void) { return 1 * 10000 + 0 * 100 + 0; }

ob_status ob_last_device_error(void* stream) {
  DeviceInfo d;
  ob_status st = current_device(&d);
  if (st != OB_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return OB_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, d.err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return OB_ERR_CUDA;
  if (word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(d.err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return OB_ERR_CUDA;
  }
  if (word & OB_DEVERR_TIMEOUT) return OB_ERR_DEVICE_TIMEOUT;
  if (word & OB_DEVERR_BOUNDS) return OB_ERR_DEVICE_BOUNDS;
  if (word & OB_DEVERR_NAN) return OB_ERR_NAN;
  return OB_OK;
}

ob_status ob_pack_signs(const float* W, int64_t N, int64_t K, uint32_t* W_packed, void* stream) {
  if (N < 0 || K < 0 || K % 32 != 0 || !elems_ok(N, K)) return OB_ERR_SHAPE;
  if (N == 0 || K == 0) return OB_OK;
  if (!W || !W_packed) return OB_ERR_NULL;
  if (misaligned(W) || misaligned(W_packed)) return OB_ERR_ALIGN;
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  return status_of(launch_pack_signs(W, N, K, W_packed, c));
}

size_t ob_svid_workspace_size(int64_t N, int64_t K) {
  if (N < 0 || K < 0 || !elems_ok(N, K)) return 0;
  return svid_workspace_bytes(N, K);
}

ob_status ob_svid_rank1(const float* W, int64_t N, int64_t K, float* a, float* b, float* sigma1, int max_iters,
                        float tol, int* iters_out, void* workspace, size_t ws_bytes, void* stream) {
  if (iters_out) *iters_out = 0;
  if (N < 0 || K < 0 || K % 4 != 0 || !elems_ok(N, K)) return OB_ERR_SHAPE;
  if (N == 0 || K == 0) return OB_OK;
  if (!W || !a || !b) return OB_ERR_NULL;
  if (misaligned(W) || misaligned(a) || misaligned(b)) return OB_ERR_ALIGN;
  if (!workspace || ws_bytes < svid_workspace_bytes(N, K)) return OB_ERR_WORKSPACE;
  if (misaligned(workspace)) return OB_ERR_ALIGN;
  if (max_iters <= 0) max_iters = 200;
  if (!(tol > 0.f)) tol = 1e-6f;
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  return run_svid(W, N, K, a, b, sigma1, max_iters, tol, iters_out, workspace, c);
}

ob_status ob_linear_ws(const void* X, int64_t M, int64_t K, const uint32_t* W_packed, int64_t N, const float* a,
                       const float* b, void* Y, int y_dtype, void* workspace, size_t ws_bytes, int path,
                       void* stream) {
  if (M < 0 || N < 0 || K < 0 || K % 32 != 0) return OB_ERR_SHAPE;
  if (!elems_ok(M, K) || !elems_ok(N, K) || !elems_ok(M, N)) return OB_ERR_SHAPE;
  if (y_dtype != OB_OUT_BF16 && y_dtype != OB_OUT_F32) return OB_ERR_UNSUPPORTED;
  if (path < 0 || (path & ~0xFF & ~OB_FLAG_STATIC_WEIGHTS) != 0) return OB_ERR_UNSUPPORTED;
  const int static_w = (path & OB_FLAG_STATIC_WEIGHTS) ? 1 : 0;
  path &= 0xFF;
  if (path > OB_PATH_TC1 || path == 2 || path == OB_PATH_STACK) return OB_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return OB_OK;
  if (!Y || !a) return OB_ERR_NULL;
  if (K > 0 && (!X || !W_packed || !b)) return OB_ERR_NULL;
  if (misaligned(Y) || misaligned(a) || (K > 0 && (misaligned(X) || misaligned(W_packed) || misaligned(b))))
    return OB_ERR_ALIGN;
  if (workspace && misaligned(workspace)) return OB_ERR_ALIGN;
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  if (K == 0) return zero_output(Y, M, N, y_dtype, c.stream);
  SignGemmArgs g{static_cast<const uint16_t*>(X), M, K, W_packed, N, b, a, Y, N, y_dtype};
  g.static_w = static_w;
  // Few output tiles on the one-CTA tcgen05 GEMM (AUTO above the decode sizes where the CTA
  // pair does not apply, OB_PATH_TC likewise, OB_PATH_TC1): split over K through the
  // workspace when it holds the partial sums.  Measured on B200 at M = 256, K = N = 4096:
  // 32 tiles on 32 SMs unsplit.
  const bool one_cta = path == OB_PATH_TC1 ||
                       ((path == OB_PATH_TC || (path == OB_PATH_AUTO && M > kDecodeMaxM)) &&
                        !sign_gemm_tc2_supported(g));
  if (one_cta && workspace) {
    const int ks = linear_split_k(M, N, K, c.num_sms);
    if (ks > 1 && ws_bytes >= (size_t)ks * (size_t)M * (size_t)N * 4)
      return status_of(launch_sign_gemm_tc_splitk(g, ks, static_cast<float*>(workspace), c));
  }
  return run_sign_gemm(g, path, c);
}

size_t ob_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0 || !elems_ok(M, K) || !elems_ok(N, K) || !elems_ok(M, N)) return 0;
  if (M == 0 || N == 0 || K == 0) return 0;
  const int ks = linear_split_k(M, N, K, sms_for_sizing());
  return ks > 1 ? align256((size_t)ks * (size_t)M * (size_t)N * 4) : 0;
}

ob_status ob_linear_ex(const void* X, int64_t M, int64_t K, const uint32_t* W_packed, int64_t N, const float* a,
                       const float* b, void* Y, int y_dtype, int path, void* stream) {
  return ob_linear_ws(X, M, K, W_packed, N, a, b, Y, y_dtype, nullptr, 0, path, stream);
}

ob_status ob_linear(const void* X, int64_t M, int64_t K, const uint32_t* W_packed, int64_t N, const float* a,
                    const float* b, void* Y, int y_dtype, void* stream) {
  return ob_linear_ex(X, M, K, W_packed, N, a, b, Y, y_dtype, OB_PATH_AUTO, stream);
}

ob_status ob_linear_ln(const void* X, int64_t M, int64_t K, const uint32_t* W_packed, int64_t N, const float* a,
                       const float* b, void* Z, int z_dtype, float eps, int path, void* stream) {
  if (!(eps >= 0.f) || eps > 3.0e38f) return OB_ERR_UNSUPPORTED;  // negative, NaN or infinite
  if (M > 2147483647) return OB_ERR_SHAPE;                         // one CTA per row
  ob_status st = ob_linear_ex(X, M, K, W_packed, N, a, b, Z, z_dtype, path, stream);
  if (st != OB_OK || M == 0 || N == 0) return st;
  LaunchCtx c;
  st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  return launch_layernorm_rows(Z, M, N, N, z_dtype, eps, c) == cudaSuccess ? OB_OK : OB_ERR_CUDA;
}

size_t ob_stack_workspace_size(void) { return 256; }

size_t ob_linear_stack_workspace_size(const ob_layer* layers, int n_layers, int64_t M) {
  const size_t base = ob_stack_workspace_size();
  if (!layers || n_layers <= 0 || M < 1 || M > kStackI8MaxM) return base;
  std::vector<StackLayerHost> host((size_t)n_layers);
  for (int i = 0; i < n_layers; ++i) {
    const ob_layer& L = layers[i];
    if (L.K < 32 || L.N < 1 || L.N > ((int64_t)1 << 35) || !elems_ok(L.N, L.K)) return base;
    host[i] = StackLayerHost{L.X, L.W_packed, L.b, L.a, L.Y, L.K, L.N, L.y_dtype, L.after_previous ? 1 : 0};
  }
  return base + align256(stack_tag_words(host.data(), n_layers, M) * sizeof(uint32_t));
}

ob_status ob_linear_stack_ex(const ob_layer* layers, int n_layers, int64_t M, void* workspace, size_t ws_bytes,
                             int path, void* stream) {
  if (n_layers < 0 || M < 0 || M > kDecodeMaxM) return OB_ERR_SHAPE;
  if (path != OB_PATH_AUTO && path != OB_PATH_MMA_DECODE && path != OB_PATH_I8) return OB_ERR_UNSUPPORTED;
  if (path == OB_PATH_I8 && M > kStackI8MaxM) return OB_ERR_UNSUPPORTED;
  if (n_layers == 0 || M == 0) return OB_OK;
  if (!layers) return OB_ERR_NULL;
  if (!workspace) return OB_ERR_NULL;
  if (misaligned(workspace)) return OB_ERR_ALIGN;
  if (ws_bytes < ob_stack_workspace_size()) return OB_ERR_WORKSPACE;
  std::vector<StackLayerHost> host((size_t)n_layers);
  for (int i = 0; i < n_layers; ++i) {
    const ob_layer& L = layers[i];
    if (L.K < 32 || L.K % 32 != 0 || L.N < 1 || L.N > ((int64_t)1 << 35) || !elems_ok(L.N, L.K))
      return OB_ERR_SHAPE;
    if (L.y_dtype != OB_OUT_BF16 && L.y_dtype != OB_OUT_F32) return OB_ERR_UNSUPPORTED;
    if (!L.X || !L.W_packed || !L.a || !L.Y) return OB_ERR_NULL;
    if (misaligned(L.X) || misaligned(L.W_packed) || misaligned(L.a) || misaligned(L.Y) ||
        (L.b && misaligned(L.b)))
      return OB_ERR_ALIGN;
    host[i] = StackLayerHost{L.X, L.W_packed, L.b, L.a, L.Y, L.K, L.N, L.y_dtype, L.after_previous ? 1 : 0};
  }
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  if (path == OB_PATH_AUTO) path = M <= kStackI8MaxM ? OB_PATH_I8 : OB_PATH_MMA_DECODE;
  // A workspace beyond the barrier words holds the tagged outputs of the dataflow form.
  const size_t base = ob_stack_workspace_size();
  uint32_t* tags = nullptr;
  size_t tag_words = 0;
  if (path == OB_PATH_I8 && ws_bytes > base) {
    tags = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + base);
    tag_words = (ws_bytes - base) / sizeof(uint32_t);
  }
  return status_of(
      launch_sign_stack(host.data(), n_layers, M, static_cast<unsigned*>(workspace), c, path, tags, tag_words));
}

ob_status ob_linear_stack(const ob_layer* layers, int n_layers, int64_t M, void* workspace, size_t ws_bytes,
                          void* stream) {
  return ob_linear_stack_ex(layers, n_layers, M, workspace, ws_bytes, OB_PATH_AUTO, stream);
}

// Bytes of the bf16 intermediate T: the smallest workspace dbf_linear accepts.
size_t dbf_t_bytes(int64_t M, int64_t r) { return align256((size_t)M * (size_t)r * 2); }

// Bytes after T that hold the grid-barrier word of the one-launch decode chain; fp32
// partial sums of a split product start after them.
constexpr size_t kDbfBarrierBytes = 256;

// K slices of DBF's first product (T = ... S_B^T, M x r, over K) when it runs on the tcgen05
// GEMM; sizing does not know K, so it takes the most slices any K allows.
int dbf_split_k(int64_t M, int64_t r, int num_sms, int64_t K = (int64_t)1 << 20) {
  return M > kDecodeMaxM ? tc_split_k(M, r, K, num_sms) : 1;
}

size_t dbf_workspace_size(int64_t M, int64_t r) {
  if (M < 0 || r < 0 || !elems_ok(M, r)) return 0;
  if (M == 0 || r == 0) return 0;  // nothing to hold
  const int ks = dbf_split_k(M, r, sms_for_sizing());
  return dbf_t_bytes(M, r) + kDbfBarrierBytes + (ks > 1 ? align256((size_t)ks * (size_t)M * (size_t)r * 4) : 0);
}

ob_status dbf_linear_ex(const void* X, int64_t M, int64_t K, const uint32_t* SB_packed, int64_t r, const float* m,
                        const uint32_t* SA_packed, int64_t N, const float* a, const float* b, void* Y, int y_dtype,
                        void* workspace, size_t ws_bytes, int path, void* stream) {
  if (M < 0 || N < 0 || K < 0 || r < 0 || K % 32 != 0 || r % 32 != 0) return OB_ERR_SHAPE;
  if (!elems_ok(M, K) || !elems_ok(r, K) || !elems_ok(M, r) || !elems_ok(N, r) || !elems_ok(M, N))
    return OB_ERR_SHAPE;
  if (y_dtype != OB_OUT_BF16 && y_dtype != OB_OUT_F32) return OB_ERR_UNSUPPORTED;
  if (path < 0 || (path & ~0xFF & ~OB_FLAG_STATIC_WEIGHTS) != 0) return OB_ERR_UNSUPPORTED;
  const int static_w = (path & OB_FLAG_STATIC_WEIGHTS) ? 1 : 0;
  path &= 0xFF;
  if (path > OB_PATH_STACK || path == 2) return OB_ERR_UNSUPPORTED;
  if (path == OB_PATH_STACK && M > kDecodeMaxM) return OB_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return OB_OK;
  if (!Y || !a) return OB_ERR_NULL;
  const bool empty_sum = (K == 0 || r == 0);
  if (!empty_sum && (!X || !SB_packed || !m || !SA_packed || !b)) return OB_ERR_NULL;
  if (misaligned(Y) || misaligned(a)) return OB_ERR_ALIGN;
  if (!empty_sum && (misaligned(X) || misaligned(SB_packed) || misaligned(m) || misaligned(SA_packed) ||
                     misaligned(b)))
    return OB_ERR_ALIGN;
  if (!empty_sum) {
    if (!workspace || ws_bytes < dbf_t_bytes(M, r)) return OB_ERR_WORKSPACE;
    if (misaligned(workspace)) return OB_ERR_ALIGN;
  }
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  if (empty_sum) return zero_output(Y, M, N, y_dtype, c.stream);
  // T = ((X ⊙ b^T) S_B^T) ⊙ m^T, rounded once to bf16, then Y = (T S_A^T) ⊙ a^T.
  uint16_t* T = static_cast<uint16_t*>(workspace);
  const size_t t_bytes = dbf_t_bytes(M, r);
  // OB_PATH_STACK (M <= 16): both products in one persistent launch of the layer-stack
  // kernels (two layers, a grid barrier between them); the barrier word sits after T in the
  // workspace.  AUTO at decode sizes takes two per-call kernels instead, chained by
  // programmatic launch: measured on B200 at M = 1, K = N = 4096, r = 2048, 6.3 us per call
  // with static weights against 16.4 us for the one launch; T (a few KB) stays in L2 either way.
  if (path == OB_PATH_STACK) {
    if (ws_bytes < t_bytes + kDbfBarrierBytes) return OB_ERR_WORKSPACE;
    const StackLayerHost two[2] = {{X, SB_packed, b, m, T, K, r, OB_OUT_BF16, 0},
                                   {T, SA_packed, nullptr, a, Y, r, N, y_dtype, 1}};
    unsigned* bar = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + t_bytes);
    return status_of(
        launch_sign_stack(two, 2, M, bar, c, M <= kStackI8MaxM ? OB_PATH_I8 : OB_PATH_MMA_DECODE));
  }
  SignGemmArgs g1{static_cast<const uint16_t*>(X), M, K, SB_packed, r, b, m, T, r, OB_OUT_BF16};
  g1.static_w = static_w;  // S_B, b, m
  // Few output tiles (small M x r): split the first product over K into fp32 partial
  // sums after T in the workspace, when the workspace holds them.
  const bool tc1 = path == OB_PATH_TC || (path == OB_PATH_AUTO && M > kDecodeMaxM && K <= sign_gemm_tc_max_k());
  const int ks = tc1 ? dbf_split_k(M, r, c.num_sms, K) : 1;
  const size_t part_off = t_bytes + kDbfBarrierBytes;
  if (ks > 1 && ws_bytes >= part_off + (size_t)ks * (size_t)M * (size_t)r * 4) {
    g1.l2_prefetch = 0;
    st = status_of(launch_sign_gemm_tc_splitk(
        g1, ks, reinterpret_cast<float*>(static_cast<char*>(workspace) + part_off), c));
  } else {
    st = run_sign_gemm(g1, path, c);
  }
  if (st != OB_OK) return st;
  SignGemmArgs g2{T, M, r, SA_packed, N, nullptr, a, Y, N, y_dtype};
  g2.static_w = static_w;  // S_A, a (T is the previous kernel's output: read after the wait)
  // The second product (K = r) splits the same way when the region after T also holds
  // its partial sums (the first product's are consumed before it runs), unless the
  // CTA-pair kernel takes it and r < 4096: measured at M = 512 on B200, r = 2048
  // unsplit on the pair kernel 42.6 us per layer against 44.7 split, r = 4704 split
  // 64.4 against 67.6 unsplit.
  const bool tc2 = path == OB_PATH_TC || (path == OB_PATH_AUTO && M > kDecodeMaxM && r <= sign_gemm_tc_max_k());
  const bool pair2 = sign_gemm_tc2_supported(g2) && r < 4096;
  const int ks2 = (tc2 && !pair2 && M > kDecodeMaxM)
                      ? tc_split_k(M, N, r, c.num_sms)
                      : 1;
  if (ks2 > 1 && ws_bytes >= part_off + (size_t)ks2 * (size_t)M * (size_t)N * 4)
    return status_of(launch_sign_gemm_tc_splitk(
        g2, ks2, reinterpret_cast<float*>(static_cast<char*>(workspace) + part_off), c));
  return run_sign_gemm(g2, path, c);
}

ob_status dbf_linear(const void* X, int64_t M, int64_t K, const uint32_t* SB_packed, int64_t r, const float* m,
                     const uint32_t* SA_packed, int64_t N, const float* a, const float* b, void* Y, int y_dtype,
                     void* workspace, size_t ws_bytes, void* stream) {
  return dbf_linear_ex(X, M, K, SB_packed, r, m, SA_packed, N, a, b, Y, y_dtype, workspace, ws_bytes,
                       OB_PATH_AUTO, stream);
}

ob_status dbf_linear_noalloc(const void* X, int64_t M, int64_t K, const uint32_t* SB_packed, int64_t r,
                             const float* m, const uint32_t* SA_packed, int64_t N, const float* a, const float* b,
                             void* Y, int y_dtype, void* stream) {
  // Size check first, before any CUDA call: the intermediate is M x r bf16.  Checked by
  // division so that no product of the sizes can wrap.
  if (M < 0 || r < 0) return OB_ERR_SHAPE;
  if (r > 0 && M > (int64_t)(OB_DBF_NOALLOC_SCRATCH_BYTES / 2) / r) return OB_ERR_WORKSPACE;
  // Device address of the static scratch on the current device, looked up once per
  // device with that device current.  The array's name in host code is only a
  // host-side handle, never a device address.
  static std::mutex mu;
  static void* scratch[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OB_ERR_CUDA;
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!scratch[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_dbf_noalloc_scratch) != cudaSuccess || p == nullptr) return OB_ERR_CUDA;
      scratch[dev] = p;
    }
    ptr = scratch[dev];
  }
  return dbf_linear_ex(X, M, K, SB_packed, r, m, SA_packed, N, a, b, Y, y_dtype, ptr,
                       (size_t)OB_DBF_NOALLOC_SCRATCH_BYTES, OB_PATH_AUTO, stream);
}

size_t dbf_factorize_workspace_size(int64_t N, int64_t K, int64_t r) {
  if (N < 1 || K < 32 || r < 32 || K % 32 != 0 || r % 32 != 0) return 0;
  if (N > kFactorizeMaxDim || K > kFactorizeMaxDim || r > kFactorizeMaxDim) return 0;
  return dbf_factorize_workspace_bytes(N, K, r);
}

ob_status dbf_factorize(const float* W, int64_t N, int64_t K, int64_t r, const float* omega, int sweeps,
                        int admm_iters, int cg_iters, float rho_rel, int refit_rounds, uint32_t* SA_packed,
                        uint32_t* SB_packed, float* a, float* m, float* b, float* history, float* best,
                        float* error, void* workspace, size_t ws_bytes, void* stream) {
  if (N < 1 || K < 32 || r < 32 || K % 32 != 0 || r % 32 != 0) return OB_ERR_SHAPE;
  if (N > kFactorizeMaxDim || K > kFactorizeMaxDim || r > kFactorizeMaxDim) return OB_ERR_SHAPE;
  if (sweeps < 0 || sweeps > 100000 || admm_iters < 1 || admm_iters > 1000 || cg_iters < 1 || cg_iters > 10000 ||
      refit_rounds < 0 || refit_rounds > 100 || !(rho_rel > 0.f) || rho_rel > 1e30f)
    return OB_ERR_UNSUPPORTED;
  if (!W || !omega || !SA_packed || !SB_packed || !a || !m || !b || !workspace) return OB_ERR_NULL;
  if (misaligned(W) || misaligned(omega) || misaligned(SA_packed) || misaligned(SB_packed) || misaligned(a) ||
      misaligned(m) || misaligned(b) || misaligned(workspace))
    return OB_ERR_ALIGN;
  if (ws_bytes < dbf_factorize_workspace_bytes(N, K, r)) return OB_ERR_WORKSPACE;
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  return run_dbf_factorize(W, N, K, r, omega, sweeps, admm_iters, cg_iters, rho_rel, refit_rounds, SA_packed,
                           SB_packed, a, m, b, history, best, error, workspace, c);
}

ob_status ob_selftest_timeout(uint64_t limit_ns, void* stream) {
  LaunchCtx c;
  ob_status st = make_ctx(stream, &c);
  if (st != OB_OK) return st;
  if (launch_timeout_selftest(limit_ns, c) != cudaSuccess) return OB_ERR_CUDA;
  return ob_last_device_error(stream);
}

}  // extern "C"
