// ob_internal.h -- host-side launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "obgemm.h"

namespace ob {

struct LaunchCtx {
  cudaStream_t stream;
  unsigned* err;   // device error word of the current device
  int num_sms;     // multiprocessors of the current device
  bool pdl;        // launch with programmatic stream serialization
  bool l2_prefetch;  // with pdl: prefetch the weights into L2 before waiting on the previous grid
};

// High half of a tagged output word (kTagMark | bf16 bits) of the dataflow form of the
// int8 layer stack; its tag area is zeroed before every launch, so a zero word is not ready.
constexpr uint32_t kTagMark = 0xA5A50000u;

// One sign-product layer  Y[m, n] = oscale[n] * sum_k (x[m, k] * iscale[k]) * s[n, k],
// with s the packed sign matrix (R x K, R = output features).  X is bf16 M x K
// (row stride K); iscale may be null (no input scale).  Y is M x R with row
// stride ldy, bf16 or fp32.
struct SignGemmArgs {
  const uint16_t* X;
  int64_t M, K;
  const uint32_t* S;
  int64_t R;
  const float* iscale;  // [K] or null
  const float* oscale;  // [R]
  void* Y;
  int64_t ldy;
  int y_dtype;          // ob_out_dtype
  int l2_prefetch;      // set by the dispatcher: prefetch this launch's weights into L2 first
  int static_w;         // S, iscale and oscale were not written by the previous grid in the
                        // stream: kernels may read them before the programmatic-launch wait
};

cudaError_t launch_pack_signs(const float* W, int64_t N, int64_t K, uint32_t* out, const LaunchCtx& c);

cudaError_t launch_sign_gemm_simt(const SignGemmArgs& g, const LaunchCtx& c);
cudaError_t launch_sign_gemm_mma_decode(const SignGemmArgs& g, const LaunchCtx& c);
// int8 tensor-core sign product for one or two tokens per pass (linear_i8.cu, i8_block.cuh).
cudaError_t launch_sign_gemm_i8(const SignGemmArgs& g, const LaunchCtx& c);
cudaError_t launch_sign_gemm_tc(const SignGemmArgs& g, const LaunchCtx& c);
// cuTensorMapEncodeTiled from the driver (null if unavailable).
void* tensor_map_encode_tiled_fn();

// The CTA-pair tcgen05 GEMM (linear_tc2.cu): bf16 Y with 16-byte-aligned rows,
// K <= 16384, M >= 512, R >= 256.
bool sign_gemm_tc2_supported(const SignGemmArgs& g);
cudaError_t launch_sign_gemm_tc2(const SignGemmArgs& g, const LaunchCtx& c);
// Whether launch_sign_gemm_tc2 takes 128-token pair tiles for this shape.
bool sign_gemm_tc2_narrow(const SignGemmArgs& g, int num_sms);

// Largest K the tcgen05 GEMM takes (its input-scale pairs live in shared memory).
int64_t sign_gemm_tc_max_k();
// K slices for the tcgen05 GEMM of an M x R output: more than one when the output has
// fewer 128 x 256 tiles than half the SMs (at most 8).
int tc_split_k(int64_t M, int64_t R, int64_t K, int num_sms);
// The tcgen05 GEMM split over K: fp32 partial sums of each slice into part
// (ksplit x M x R floats), then a reduction that applies oscale and writes Y.
// Slices hold at least 1024 k; falls back to the unsplit kernel when K is too short for
// two slices or R, ldy are not multiples of 4.
cudaError_t launch_sign_gemm_tc_splitk(const SignGemmArgs& g, int ksplit, float* part, const LaunchCtx& c);

// SVID power iteration pieces (see svid.cu).
size_t svid_workspace_bytes(int64_t N, int64_t K);
ob_status run_svid(const float* W, int64_t N, int64_t K, float* a, float* b, float* sigma1, int max_iters,
                   float tol, int* iters_out, void* ws, const LaunchCtx& c);

cudaError_t launch_timeout_selftest(uint64_t limit_ns, const LaunchCtx& c);

// DBF factorisation (dbf_factorize.cu): workspace bytes, and the whole run (synchronous;
// arguments validated by the caller).  history / best_out / error_out are host pointers
// (nullable).
size_t dbf_factorize_workspace_bytes(int64_t N, int64_t K, int64_t r);
ob_status run_dbf_factorize(const float* W, int64_t N, int64_t K, int64_t r, const float* omega, int sweeps,
                            int admm_iters, int cg_iters, float rho_rel, int refit_rounds, uint32_t* SA_packed,
                            uint32_t* SB_packed, float* a, float* m, float* b, float* history, float* best_out,
                            float* error_out, void* workspace, const LaunchCtx& lc);

// One layer of a persistent layer-stack launch (linear_stack.cu).
struct StackLayerHost {
  const void* X;        // bf16 [M, K]
  const uint32_t* S;    // packed [N, K/32]
  const float* iscale;  // [K] or null
  const float* oscale;  // [N]
  void* Y;              // [M, N]
  int64_t K, N;
  int y_dtype;
  int barrier;          // reads an output of an earlier layer of the list
};
// Runs the list (M <= 16) as cooperative launches of at most stack_max_layers_per_launch()
// layers; bar: 8 bytes of device memory (zeroed by the launcher).  path: OB_PATH_I8 (M <= 2)
// for the int8 form, OB_PATH_MMA_DECODE for the bf16 form.
// tags / tag_words: device area for tagged outputs (dataflow launches of the int8 form, where
// stack_tag_words() says the list allows them), or null / 0 for grid barriers only.
cudaError_t launch_sign_stack(const StackLayerHost* layers, int n, int64_t M, unsigned* bar, const LaunchCtx& c,
                              int path, uint32_t* tags = nullptr, size_t tag_words = 0);
int stack_max_layers_per_launch();
// 32-bit words of tagged outputs a dataflow launch of the list needs (the largest over its
// launches), or 0 when no launch of it qualifies (one token only): every layer writes its own buffer, and
// every input is either outside all outputs of its launch or exactly the bf16 output of an
// earlier layer of it.
size_t stack_tag_words(const StackLayerHost* layers, int n, int64_t M);

// Z = LayerNorm(Y) per row of the M x N matrix Y (row stride ld elements), in place.
cudaError_t launch_layernorm_rows(void* Y, int64_t M, int64_t N, int64_t ld, int y_dtype, float eps,
                                  const LaunchCtx& c);

// Largest M handled by one pass of the tensor-memory decode kernel.
constexpr int kDecodeMaxM = 16;

}  // namespace ob
