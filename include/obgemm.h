/*
 * obgemm.h -- C ABI of libobgemm.so: sign-only-weight linear layers on B200 (sm_100a).
 *
 * Two layer forms share one packed sign format:
 *
 *   OneBit  Y = [(X ⊙ b^T) · W_sign^T] ⊙ a^T
 *           "1bit量化" (blog.zerodtree.com), notes on "OneBit: Towards Extremely
 *           Low-bit Large Language Models": section "rank-1 approximation"
 *           (W = W_sign ⊙ |W|, |W| ≈ a b^T) and "proposition 1".  The page
 *           assigns b^T to the layer's input scale g and a^T to its output
 *           scale h.
 *
 *   DBF     Y = ((((X ⊙ b^T) · S_B^T) ⊙ m^T) · S_A^T) ⊙ a^T
 *           "Addition is almost all you need: Compressing large language models
 *           with double binary factorization" (gist.science), section
 *           "Methodologie: Double Binary Factorization (DBF)", the factorised
 *           weight W ≈ (a ⊙ A ⊙ m^T)(B ⊙ b^T) and its inference chain.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Matrices are dense and row-major.  W is N x K (out x in), X is M x K,
 *    Y is M x N.  Index names follow the pages: a has length N (output scale),
 *    b has length K (input scale); for DBF, S_A is N x r, S_B is r x K, m has
 *    length r.
 *  - Packed sign format: row n of an R x C sign matrix is C/32 uint32 words;
 *    bit i of word w holds column 32*w + i (least significant bit first), and
 *    a set bit means -1, a clear bit +1.  Sign(w) = -1 exactly when w < 0, so
 *    +0.0 and -0.0 pack as +1 (the pages leave Sign(0) open).  C must be a
 *    multiple of 32.
 *  - X is bf16 (IEEE bfloat16 bit patterns, passed as const void*), scale
 *    vectors are fp32, Y is bf16 (round to nearest even) or fp32 by `y_dtype`.
 *  - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *    owns every buffer; the library allocates no device memory.  It holds
 *    one 4-byte device error word per device (module-scope) and the static
 *    scratch array of dbf_linear_noalloc (OB_DBF_NOALLOC_SCRATCH_BYTES per
 *    device, module-scope), and nothing else.  Every device pointer must be
 *    16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous and stream-ordered unless noted.
 *  - Errors: argument checks run on the host before any launch and return a
 *    status without launching.  Launch failures return OB_ERR_CUDA.  Faults
 *    found on the device (a bounded wait that ran out, NaN in an input that
 *    must be finite) set the device error word, which ob_last_device_error()
 *    reads.  No call aborts or throws across the ABI.
 *  - Empty problems (M == 0 or N == 0) return OB_OK and touch nothing; K == 0
 *    (or r == 0 for DBF) writes Y = 0.
 */
#ifndef OBGEMM_H_
#define OBGEMM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define OB_API __attribute__((visibility("default")))
#else
#define OB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ob_status {
  OB_OK = 0,
  OB_ERR_NULL = 1,            /* a required pointer is NULL */
  OB_ERR_SHAPE = 2,           /* negative size, or K / r not a multiple of 32 */
  OB_ERR_ALIGN = 3,           /* a pointer is not 16-byte aligned */
  OB_ERR_NAN = 4,             /* NaN in an input that must be finite */
  OB_ERR_NOT_CONVERGED = 5,   /* SVID hit max_iters before the tolerance */
  OB_ERR_WORKSPACE = 6,       /* workspace NULL or smaller than required */
  OB_ERR_CUDA = 7,            /* a CUDA runtime call or kernel launch failed */
  OB_ERR_DEVICE_TIMEOUT = 8,  /* a bounded wait inside a kernel ran out */
  OB_ERR_UNSUPPORTED = 9,     /* device is not sm_100, an option is unknown, or OB_PATH_TC with K > 32768 */
  OB_ERR_DEVICE_BOUNDS = 10   /* a kernel's own bounds check refused an access */
} ob_status;

typedef enum ob_out_dtype {
  OB_OUT_BF16 = 0,
  OB_OUT_F32 = 1
} ob_out_dtype;

/* Kernel choice for ob_linear_ex / dbf_linear_ex / ob_linear_stack_ex.  Value 2 is not used
 * (it named a tensor-memory decode kernel that measured slower than every other path and
 * was removed); passing it returns OB_ERR_UNSUPPORTED. */
typedef enum ob_path {
  OB_PATH_AUTO = 0,        /* M == 1: OB_PATH_SIMT; M <= 16 or K > 32768: OB_PATH_MMA_DECODE; else OB_PATH_TC */
  OB_PATH_SIMT = 1,        /* CUDA-core mat-vec: one token by table lookup, more tokens by select/add */
  OB_PATH_TC = 3,          /* tcgen05 tiled GEMM for large M (activations by TMA); K <= 32768; a
                              2-CTA (cta_group::2) tile where bf16 Y, M >= 512, N >= 256, K <= 16384,
                              else one CTA per tile */
  OB_PATH_MMA_DECODE = 4,  /* bf16 warp-level MMA, signs unpacked in registers, M <= 16 per pass */
  OB_PATH_I8 = 5,          /* int8 warp-level MMA (u8 x s8 -> s32): each packed word becomes eight operand
                              registers with one AND each, activations quantised per token to 21 bits in
                              three 7-bit limbs, exact integer sums; M <= 2 per pass */
  OB_PATH_STACK = 6,       /* dbf_linear_ex only, M <= 16: both sign products in one persistent launch of
                              the layer-stack kernel, a grid barrier between them */
  OB_PATH_TC1 = 7          /* ob_linear_ex / ob_linear_ln only: the one-CTA tcgen05 GEMM even where
                              OB_PATH_TC would take the CTA pair (tests, measurement); K <= 32768 */
} ob_path;

/* Flag OR-ed into the path argument of ob_linear_ex (and ob_linear_ln): the caller
 * guarantees that W_packed, a and b were not written by the kernel launched just before
 * this call on the same stream (weights loaded once and used by call after call).  The
 * one-token kernel (its sign words and output scales) and the warp-MMA decode kernel (its
 * first chunk of sign words) then start reading before waiting for that kernel to finish
 * (programmatic dependent launch), so the weights stream in while it runs.  The other
 * kernels ignore the flag.  Any other bit above the low 8 is rejected with
 * OB_ERR_UNSUPPORTED. */
#define OB_FLAG_STATIC_WEIGHTS 0x100

/* Human-readable name of a status code (static string, never NULL). */
OB_API const char* ob_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
OB_API int ob_version(void);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns OB_OK, OB_ERR_DEVICE_TIMEOUT, OB_ERR_DEVICE_BOUNDS
 * or OB_ERR_NAN (highest severity first), or OB_ERR_CUDA if the
 * synchronisation itself fails.
 */
OB_API ob_status ob_last_device_error(void* stream);

/*
 * Sign extraction and packing, W_sign = Sign(W)
 * ("1bit量化", section "rank-1 approximation": W = W_sign ⊙ |W|; the layer's
 *  W_±1 = Sign(W) in the distillation section).
 *   W         device, fp32 N x K, row-major; must be free of NaN.
 *   W_packed  device, uint32 N x (K/32), written in the packed sign format.
 * K % 32 == 0.  A NaN in W packs as +1 and sets OB_ERR_NAN in the device
 * error word.  Asynchronous.
 */
OB_API ob_status ob_pack_signs(const float* W, int64_t N, int64_t K, uint32_t* W_packed, void* stream);

/* Bytes of device workspace ob_svid_rank1 needs for an N x K matrix. */
OB_API size_t ob_svid_workspace_size(int64_t N, int64_t K);

/*
 * Rank-1 SVID of |W|: |W| ≈ a b^T with a = sqrt(sigma1) u1, b = sqrt(sigma1) v1,
 * (u1, sigma1, v1) the leading singular triple of |W|, both vectors
 * nonnegative ("1bit量化", section "rank-1 approximation"; the page takes the
 * triple from an SVD, this routine finds it by power iteration on |W|^T |W|).
 *   W          device, fp32 N x K, K % 4 == 0.
 *   a          device, fp32 [N] (output scale, the page's h).
 *   b          device, fp32 [K] (input scale, the page's g).
 *   sigma1     device, fp32 [1], or NULL.
 *   max_iters  iteration cap (<= 0 selects 200).
 *   tol        stop when ||v_t - v_{t-1}||_2 <= tol (<= 0 selects 1e-6).
 *   iters_out  HOST int, or NULL: iterations taken.
 *   workspace  device, at least ob_svid_workspace_size(N, K) bytes.
 * The stopping test runs on the device; the host queues 8 iterations at a time and
 * synchronises `stream` once per 8 (once in all when the iteration converges within
 * 8, as it does on the workloads in 3); it is an offline conversion.
 * Returns OB_ERR_NOT_CONVERGED with the last iterate written if the cap is
 * reached, OB_ERR_NAN if W holds NaN.  An all-zero W gives a = b = 0,
 * sigma1 = 0 and OB_OK.
 */
OB_API ob_status ob_svid_rank1(const float* W, int64_t N, int64_t K,
                        float* a, float* b, float* sigma1,
                        int max_iters, float tol, int* iters_out,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * OneBit linear layer, Proposition 1: Y = [(X ⊙ b^T) · W_sign^T] ⊙ a^T
 * ("1bit量化", section "proposition 1").
 *   X         device, bf16 M x K.
 *   W_packed  device, uint32 N x (K/32), packed sign format.
 *   a         device, fp32 [N] (the page's h).
 *   b         device, fp32 [K] (the page's g).
 *   Y         device, M x N, bf16 or fp32 by y_dtype.
 * K % 32 == 0.  Accumulates in fp32.  Asynchronous.  OB_PATH_AUTO picks the
 * table-driven CUDA-core kernel for M == 1, the warp-level MMA decode kernel for
 * M <= 16 (and for K > 32768) and the tiled tcgen05 GEMM above.
 */
OB_API ob_status ob_linear(const void* X, int64_t M, int64_t K,
                    const uint32_t* W_packed, int64_t N,
                    const float* a, const float* b,
                    void* Y, int y_dtype, void* stream);

/* Bytes of device workspace ob_linear_ws can use for an M x K -> N layer: fp32 partial
 * sums (slices x M x N x 4 bytes) when the layer would run on the one-CTA tcgen05 GEMM with
 * fewer output tiles than half the SMs of the current device (e.g. M = 256, K = N = 4096),
 * N % 4 == 0 and K holds at least two slices of 1024; 0 when no split applies.  An upper
 * bound: the output dtype is not known here, and a bf16 layer that the CTA pair takes
 * (M >= 512, N >= 256, K <= 16384) runs unsplit. */
OB_API size_t ob_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * ob_linear_ex with a caller workspace.  Where the layer runs on the one-CTA tcgen05 GEMM
 * (OB_PATH_AUTO above 16 tokens when the CTA pair does not apply, OB_PATH_TC likewise,
 * OB_PATH_TC1) with few output tiles, K is split into slices whose fp32 partial sums go to
 * the workspace; a second kernel sums them, applies a and stores Y.  A workspace smaller than
 * ob_linear_workspace_size (or NULL with ws_bytes 0) runs unsplit.
 *   workspace  device, 16-byte aligned, or NULL; not shared with a concurrent call.
 * Otherwise as ob_linear_ex.
 */
OB_API ob_status ob_linear_ws(const void* X, int64_t M, int64_t K,
                       const uint32_t* W_packed, int64_t N,
                       const float* a, const float* b,
                       void* Y, int y_dtype, void* workspace, size_t ws_bytes, int path, void* stream);

/* ob_linear with an explicit kernel choice (ob_path). */
OB_API ob_status ob_linear_ex(const void* X, int64_t M, int64_t K,
                       const uint32_t* W_packed, int64_t N,
                       const float* a, const float* b,
                       void* Y, int y_dtype, int path, void* stream);

/*
 * OneBit layer followed by LayerNorm: Z = LayerNorm(Y), Y as in ob_linear
 * ("1bit量化", knowledge-distillation section: the student's Y is followed by
 * Z = LayerNorm(Y)).  Per token (a row of Y), over its N features:
 * z = (y - mean) / sqrt(var + eps), var the biased variance, no affine parameters
 * (the page shows none).
 *   Z      device, M x N, bf16 or fp32 by z_dtype; Y is computed into Z and
 *          normalised in place (a second kernel; statistics from the stored Y).
 *   eps    >= 0 and finite (1e-5 is the usual choice); otherwise OB_ERR_UNSUPPORTED
 *          before anything is launched.
 *   path   kernel for the linear layer, as in ob_linear_ex.
 * Other arguments and errors as ob_linear_ex.  Asynchronous.  A row with a single
 * feature, or a constant row, normalises to zeros.
 */
OB_API ob_status ob_linear_ln(const void* X, int64_t M, int64_t K,
                       const uint32_t* W_packed, int64_t N,
                       const float* a, const float* b,
                       void* Z, int z_dtype, float eps, int path, void* stream);

/*
 * One layer of ob_linear_stack: Y = [(X ⊙ b^T) · W_sign^T] ⊙ a^T as in ob_linear.
 *   X, W_packed, a, Y   device pointers as in ob_linear (X bf16 M x K, Y M x N).
 *   b                   device fp32 [K], or NULL for no input scale.
 *   K, N                K % 32 == 0, K >= 32, N >= 1.
 *   y_dtype             ob_out_dtype of Y.
 *   after_previous      nonzero if X is (or overlaps) the output of an earlier layer of
 *                       the list: every earlier layer finishes before this one starts.
 *                       Ignored for the first layer.
 */
typedef struct ob_layer {
  const void* X;
  const uint32_t* W_packed;
  const float* a;
  const float* b;
  void* Y;
  int64_t K;
  int64_t N;
  int32_t y_dtype;
  int32_t after_previous;
} ob_layer;

/* Bytes of device workspace ob_linear_stack needs (its grid-barrier counter). */
OB_API size_t ob_stack_workspace_size(void);

/*
 * Bytes of device workspace with which ob_linear_stack runs this list in its dataflow form:
 * ob_stack_workspace_size() plus M x N x 4 bytes for every layer whose output a later layer
 * of the same launch reads.  In that form (int8, M == 1) a layer also writes its output as
 * tagged 32-bit words, and a layer that reads it polls those words instead of waiting at a
 * grid barrier.  The list qualifies when every layer writes its own buffer (no two outputs
 * overlap) and every input is either outside all outputs of the list or exactly the bf16
 * output of an earlier layer; otherwise (and for M > 1) this returns
 * ob_stack_workspace_size(), and the list runs with grid barriers.  The library zeroes the
 * tag area before every launch.
 */
OB_API size_t ob_linear_stack_workspace_size(const ob_layer* layers, int n_layers, int64_t M);

/*
 * A list of OneBit layers at M <= 16 tokens (decode) in one persistent cooperative
 * launch per 320 layers, instead of one launch per layer: a decoder's layers read
 * one another's outputs, and per-layer launches pay a launch and a drain for each.
 * The layers between two after_previous flags run back to back; a flagged layer
 * waits at a grid-wide barrier (bounded: a wait that runs out records
 * OB_ERR_DEVICE_TIMEOUT for ob_last_device_error and the launch ends).  The pages
 * have no counterpart: this is how their layer is applied layer after layer.
 *   layers     HOST array of n_layers descriptors (read during the call only).
 *   M          tokens, 0 <= M <= 16 (OB_ERR_SHAPE above).
 *   workspace  device, at least ob_stack_workspace_size() bytes, not shared with a
 *              concurrently running ob_linear_stack; with
 *              ob_linear_stack_workspace_size(layers, n_layers, M) bytes a qualifying list
 *              runs in the dataflow form (no grid barriers).
 * Weights and scales must not be outputs of layers of the same list.  Validation of
 * every descriptor happens before anything is launched.  Asynchronous.
 * Kernel (OB_PATH_AUTO): M <= 2, the int8 form (one contiguous range of 16-row tiles
 * per CTA and barrier group, packed signs fetched into shared memory by bulk copies ahead
 * of the grid barrier, activation limbs staged once per layer per CTA, u8 x s8 warp-level
 * MMA); M > 2, the bf16 warp-level MMA form (32-row blocks round robin).
 */
OB_API ob_status ob_linear_stack(const ob_layer* layers, int n_layers, int64_t M,
                          void* workspace, size_t ws_bytes, void* stream);

/* ob_linear_stack with an explicit form: OB_PATH_AUTO, OB_PATH_MMA_DECODE (bf16, any
 * M <= 16) or OB_PATH_I8 (M <= 2; OB_ERR_UNSUPPORTED above).  Other values:
 * OB_ERR_UNSUPPORTED. */
OB_API ob_status ob_linear_stack_ex(const ob_layer* layers, int n_layers, int64_t M,
                             void* workspace, size_t ws_bytes, int path, void* stream);

/*
 * Bytes of device workspace dbf_linear uses: the M x r bf16 intermediate T, 256 bytes
 * after it (the grid-barrier word of the OB_PATH_STACK form) and, when the first
 * product runs on the tcgen05 GEMM with fewer output tiles than half the SMs of the
 * current device (e.g. M = 512, r = 2048), fp32 partial sums for splitting it over K
 * (up to 8 x M x r x 4 bytes).  dbf_linear accepts any workspace of at least T's size
 * (M x r x 2 rounded up to 256 bytes); a smaller one than this function returns runs the
 * first product without the split (and rejects OB_PATH_STACK with OB_ERR_WORKSPACE).
 */
OB_API size_t dbf_workspace_size(int64_t M, int64_t r);

/*
 * DBF linear layer: Y = ((((X ⊙ b^T) · S_B^T) ⊙ m^T) · S_A^T) ⊙ a^T
 * ("Addition is almost all you need ...", section "Methodologie: Double Binary
 *  Factorization (DBF)", inference equation).
 *   X          device, bf16 M x K.
 *   SB_packed  device, uint32 r x (K/32): S_B (the page's B_±1).
 *   m          device, fp32 [r], middle scale.
 *   SA_packed  device, uint32 N x (r/32): S_A (the page's A_±1).
 *   a          device, fp32 [N];  b  device, fp32 [K].
 *   Y          device, M x N, bf16 or fp32 by y_dtype.
 *   workspace  device, at least dbf_workspace_size(M, r) bytes; holds the
 *              intermediate T = ((X ⊙ b^T) S_B^T) ⊙ m^T between the two sign
 *              products (it stays in L2 at the workload sizes).
 * K % 32 == 0, r % 32 == 0.  Asynchronous.  M <= 16 (decode): the two products are two
 * decode kernels chained by programmatic dependent launch; T (M x r bf16, a few KB) is
 * written to L2 and read back from it by the second.  Larger M: two tcgen05 GEMMs, the
 * first split over K when it has few output tiles.  dbf_linear_ex with OB_PATH_STACK runs
 * both products in one persistent launch instead (measured slower at decode sizes).
 */
OB_API ob_status dbf_linear(const void* X, int64_t M, int64_t K,
                     const uint32_t* SB_packed, int64_t r, const float* m,
                     const uint32_t* SA_packed, int64_t N,
                     const float* a, const float* b,
                     void* Y, int y_dtype,
                     void* workspace, size_t ws_bytes, void* stream);

/* dbf_linear with an explicit kernel choice (ob_path) for both sign products. */
OB_API ob_status dbf_linear_ex(const void* X, int64_t M, int64_t K,
                        const uint32_t* SB_packed, int64_t r, const float* m,
                        const uint32_t* SA_packed, int64_t N,
                        const float* a, const float* b,
                        void* Y, int y_dtype,
                        void* workspace, size_t ws_bytes, int path, void* stream);

/*
 * Bytes of device workspace dbf_factorize needs for W N x K and middle dimension r
 * (0 for shapes it rejects).  About 4 bytes x (5 N r + 5 K r + 3 max(N, K) r + 2 r^2
 * + N K).
 */
OB_API size_t dbf_factorize_workspace_size(int64_t N, int64_t K, int64_t r);

/*
 * DBF factorisation W ≈ diag(a) · S_A · diag(m) · S_B · diag(b) ("Addition is almost
 * all you need: Compressing large language models with double binary factorization",
 * gist.science, "Optimalisatie en Training": alternating minimisation with ADMM, the
 * binary constraints met by an SVID-based projection; the page gives no steps).  The
 * steps taken:
 *   start  A = W Ω; B = the ridge least-squares fit of W ≈ A B (ridge 0.1 trace(AᵀA)/r);
 *          each factor projected onto {diag(u) · Sign · diag(v)} by the rank-1 SVID of
 *          its magnitudes (OneBit's construction).
 *   sweep  admm_iters ADMM steps on S_A's factor, then as many on S_B's: a ridge
 *          least-squares step toward the projection (penalty rho = rho_rel · trace of
 *          the other factor's Gram matrix / r; solved by cg_iters conjugate-gradient
 *          iterations per row, warm-started: 5 reach the quality of exact solves on the
 *          cases measured), the projection, the dual update.
 *   keep   the best ||W − Z_A Z_B||_F over the start and the sweeps;
 *   refit  a, then b, then m by exact least squares with the signs fixed,
 *          refit_rounds times.
 * Unweighted: the page's importance weights need calibration data.
 *   W          device fp32 N x K, row-major.
 *   omega      device fp32 K x r: the start's random matrix (drawn by the caller).
 *   K, r       multiples of 32 (the packed word), r >= 32; N >= 1; each at most 2^22.
 *   SA_packed  device N x r/32 words, SB_packed device r x K/32 words: the signs in
 *              the layout of ob_pack_signs (bit = 1 <=> -1), ready for dbf_linear.
 *   a, m, b    device fp32 [N], [r], [K] (refitted scales may be negative).
 *   history    host fp32 [sweeps], ||W − Z_A Z_B||_F after each sweep (nullable);
 *   best       host fp32, the kept iterate's error (nullable);
 *   error      host fp32, the error after the refit (nullable).
 *   workspace  device, at least dbf_factorize_workspace_size(N, K, r) bytes.
 * SYNCHRONOUS: returns when the result is in place (it reads the error back after
 * every sweep).  OB_ERR_UNSUPPORTED for sweeps outside [0, 100000], admm_iters
 * outside [1, 1000], cg_iters outside [1, 10000], refit_rounds outside [0, 100] or
 * rho_rel not positive and finite; OB_ERR_NAN if W (or Ω) leads to a non-finite
 * error.  Parity with the fp64 oracle is to properties, not digits: the page's
 * method is a heuristic, and sign decisions near zero differ between precisions.
 */
OB_API ob_status dbf_factorize(const float* W, int64_t N, int64_t K, int64_t r, const float* omega, int sweeps,
                               int admm_iters, int cg_iters, float rho_rel, int refit_rounds,
                               uint32_t* SA_packed, uint32_t* SB_packed, float* a, float* m, float* b,
                               float* history, float* best, float* error, void* workspace, size_t ws_bytes,
                               void* stream);

/* Size of the static scratch behind dbf_linear_noalloc: M * r * 2 bytes must fit. */
#define OB_DBF_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/*
 * dbf_linear for callers that cannot allocate device memory (the pages have no
 * counterpart; this is a deployment convenience).  Same operation, arguments
 * and result as dbf_linear, minus the workspace: the M x r intermediate lives
 * in a static device array of OB_DBF_NOALLOC_SCRATCH_BYTES that the library
 * reserves on every GPU where it is loaded, for the life of the process.
 *
 * Who needs it: code that enqueues work while its stream is being captured
 * into a CUDA graph (cudaMalloc is not a stream operation, cannot be recorded,
 * and may synchronise the device, which capture forbids); inference engines
 * and framework plugins that run against a fixed memory plan and may not
 * allocate at enqueue time; and callers whose device memory is owned by
 * another allocator that a raw cudaMalloc would bypass.  This call itself
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *
 * The array holds only the intermediate, so the first product never takes the
 * split over K that dbf_linear uses when its workspace also holds fp32 partial
 * sums (M = 512, r = 2048 is such a case): there this call runs that product
 * unsplit, a few microseconds slower than dbf_linear with a full workspace.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  Returns OB_ERR_WORKSPACE, launching nothing, when M * r * 2 bytes
 * exceed OB_DBF_NOALLOC_SCRATCH_BYTES.  Every call on a device shares the one
 * array and it keeps the last call's contents (each call overwrites the
 * intermediate before reading it): calls that may overlap on the GPU (other
 * streams, other host threads) race and must be serialised by the caller.
 */
OB_API ob_status dbf_linear_noalloc(const void* X, int64_t M, int64_t K,
                                    const uint32_t* SB_packed, int64_t r, const float* m,
                                    const uint32_t* SA_packed, int64_t N,
                                    const float* a, const float* b,
                                    void* Y, int y_dtype, void* stream);

/*
 * Self-test of the bounded-wait machinery (no counterpart on the pages): one
 * CTA waits on a barrier that nothing completes, first with the suspending
 * wait, then with the polling one, each giving up after `limit_ns` nanoseconds
 * (capped at 1 s); the second records OB_ERR_DEVICE_TIMEOUT in the device error
 * word and the kernel returns.  Synchronises `stream`; returns what
 * ob_last_device_error reports (OB_ERR_DEVICE_TIMEOUT when the machinery works,
 * OB_ERR_NAN if the suspending wait did not give up as it must).
 */
OB_API ob_status ob_selftest_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* OBGEMM_H_ */
