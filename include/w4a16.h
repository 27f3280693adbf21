/*
 * w4a16.h -- C ABI of the B200 (sm_100a) group-wise 4-bit weight-only
 * quantization library and its W4A16 decode GEMV / skinny GEMM.
 *
 * What is computed (pages cited by title and section):
 *
 *  - AWQ activation-aware scaling: salient input channels of the weight are
 *    multiplied by s > 1 and the activations divided by s, with s = s_X^alpha
 *    and s_X the mean activation magnitude per input channel ("MIT 6.5940
 *    Fall 2024 Lecture 13: LLM Deployment" reading guide, §AWQ, slides 25-28;
 *    "Learning-ML-DL ch. 11", §11.4).  The 1/s on the activation is folded
 *    into the previous op, so w4a16_gemm receives x already divided by s.
 *  - Round-to-nearest group quantization Q(w) = Delta * Round(w / Delta) per
 *    group of 128 input channels (Lecture 13 guide, §AWQ, slide 26), with the
 *    zero-point (asymmetric) form of the "CMU 11-868 Model Quantization"
 *    reading guide (§absmax and zero-point, lecture slide 10).
 *  - Packing the codes offline into 32-bit words so that one AND (and one
 *    shift) unpacks them (Lecture 13 guide, §TinyChat, slide 36), and a GEMV
 *    that dequantizes in registers, fused with the product (slide 37), for
 *    memory-bound batch-1 decode (§"why W8A8 is not enough", slides 19-20).
 *
 * Conventions shared by every entry point:
 *  - All tensors are dense, row-major, on the current CUDA device, owned by
 *    the caller.  The library never allocates device or host memory.
 *  - "fp16" is IEEE binary16 (__half).  Every pointer must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).  A
 *    return of W4A16_OK means the arguments were valid and the work was
 *    enqueued; nothing is launched when a negative status is returned.
 *  - Errors: a negative w4a16_status; w4a16_last_error() gives a message
 *    (thread-local, valid until the next call on the same thread).
 *
 * Packed layout v1 (our own design for sm_100a; w4a16_layout_version() == 1):
 *    qweight is uint32[N][K/8].  Word (n, j) holds the codes of
 *    k = 8j + i, i = 0..7.  Nibble slot p (bits 4p..4p+3) holds
 *    i = {0, 2, 4, 6, 1, 3, 5, 7}[p].  Hence (word >> 4t) & 0x000F000F has the
 *    codes of k = 8j+2t and 8j+2t+1 in its low and high 16-bit halves, which
 *    OR 0x64006400 turns into the fp16 pair (1024 + q0, 1024 + q1).
 *    3-bit codes use the same nibble containers.
 *    scales[n][g] = Delta and zeros[n][g] = z (an integer held in fp16) for
 *    the group g = k / group; the dequantized weight is (u - z) * Delta.
 */
#ifndef W4A16_H_
#define W4A16_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define W4A16_API __attribute__((visibility("default")))
#else
#define W4A16_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; spelled out so this header needs no CUDA headers. */
typedef struct CUstream_st* w4a16_stream_t;

typedef enum {
  W4A16_OK = 0,
  W4A16_ERR_ARG = -1,          /* null pointer, non-positive size, bad enum, non-finite alpha */
  W4A16_ERR_ALIGN = -2,        /* a pointer is not 16-byte aligned */
  W4A16_ERR_SHAPE = -3,        /* K not a multiple of the group, sizes too large */
  W4A16_ERR_UNSUPPORTED = -4,  /* valid but unsupported: group != 128, bits not in {3,4} */
  W4A16_ERR_WORKSPACE = -5,    /* workspace missing or smaller than w4a16_gemm_workspace_size */
  W4A16_ERR_CUDA = -6,         /* a CUDA runtime call or a kernel launch failed */
  W4A16_ERR_DEVICE = -7        /* a kernel gave up waiting (see w4a16_gemm_check) */
} w4a16_status;

typedef enum {
  W4A16_ASYM = 0,  /* Delta = fp16((max-min)/(2^bits-1)), z = clamp(Round(-min/Delta), 0, 2^bits-1) */
  W4A16_SYM = 1    /* Delta = fp16(max|w|/2^(bits-1)),    z = 2^(bits-1) */
} w4a16_mode;

/*
 * awq_act_scale -- per-input-channel AWQ scale from calibration activations.
 *
 *   s[k] = fp16( (mean_t |X[t][k]|) ^ alpha ),  t = 0..T-1
 *
 * s_X = mean |X| per input channel is the calibration statistic ("MIT 6.5940
 * Lab 4 + Lab 5" reading guide, §Lab 4 setup: mean |X| over 512-token blocks)
 * and s = s_X^alpha the scale (Lecture 13 guide, §AWQ, slide 28).  The mean
 * is formed in fp64 (exact, hence independent of summation order, for T <= 8192)
 * and the power in fp64; s may differ from a correctly rounded result by one fp16 ulp
 * only when s_X^alpha lies within a few fp64 ulps of an fp16 rounding boundary.
 *
 *   X     fp16 [T][K], device.      s  fp16 [K], device (output).
 *   T, K  >= 1.   alpha  finite; the pages search it in [0, 1] (any finite value accepted).
 */
W4A16_API w4a16_status awq_act_scale(const void* X, int T, int K, double alpha, void* s,
                           w4a16_stream_t stream);

/*
 * awq_quantize_pack -- AWQ scaling + group RTN + layout-v1 packing.
 *
 *   w'[n][k] = fp16(W[n][k] * s[k])               (one rounding; s == NULL means s = 1)
 *   per group (n, g) of `group` consecutive k:
 *     ASYM: Delta = fp16(fp64(max w' - min w') / (2^bits - 1)),
 *           z = clamp(Round(-min w' / Delta), 0, 2^bits - 1)
 *     SYM:  Delta = fp16(max |w'| / 2^(bits-1)),   z = 2^(bits-1)
 *     a Delta that rounds to zero is replaced by the Delta of a unit range
 *   u[n][k] = clamp(Round(w'[n][k] / Delta) + z, 0, 2^bits - 1)
 *   Round = round half to even, on the exact quotients.
 *
 *   W        fp16 [N][K], device.         s  fp16 [K] or NULL, device.
 *   qweight  uint32 [N][K/8] (output).    scales, zeros  fp16 [N][K/group] (outputs).
 *   N >= 1;  K a multiple of group;  group == 128;  bits in {3, 4}.
 *   W * s must be finite in fp16 (|W*s| <= 65504); other inputs give
 *   unspecified codes but never fault.
 * The results are bit-exact: identical on every call and to the reference
 * definition above.
 */
W4A16_API w4a16_status awq_quantize_pack(const void* W, const void* s, int N, int K, int group, int bits,
                               w4a16_mode mode, uint32_t* qweight, void* scales, void* zeros,
                               w4a16_stream_t stream);

/*
 * w4a16_gemm_workspace_size -- bytes of workspace that w4a16_gemm needs.
 * Returns 0 for invalid sizes.  The workspace holds a device status word,
 * 1024 partial-tile flags, per-row-block arrival counters and fp32 split-K
 * partial sums (M x N for M <= 4); for M >= 5 it adds, after room for the
 * M = 4 partial sums, one 128 x MP fp32 partial-tile slot per streaming
 * multiprocessor of the current device for the tensor-core path (MP, the
 * token tile, is one of 16, 32, 64, 96, 128, 192, 256: the smallest that
 * holds M).  For M > 256 it is the size for M = 256.  Everything before the
 * slots must be zero before the first call; every completed call leaves it so.
 */
W4A16_API size_t w4a16_gemm_workspace_size(int M, int N, int K, int group);

/*
 * w4a16_gemm -- y = x * dequant(qweight, scales, zeros)^T.
 *
 *   y[m][n] = fp16( sum_g Delta[n][g] * sum_{k in g} (u[n][k] - z[n][g]) * x[m][k] )
 *
 * with fp32 accumulation.  M = 1 runs on the CUDA cores (whole rows per SM, no
 * partial sums).  M = 2..8 runs on register-sourced tensor-core MMAs
 * (mma.sync, the integers u - z exact in fp16, Delta applied per group in
 * fp32) when K is a multiple of 256 and the activations of M tokens fit in
 * shared memory; otherwise M = 2..4 runs on the CUDA cores (whole rows or
 * split-K).  The rest, up to 256 tokens per launch, runs on the tcgen05 tensor
 * cores, with w_hat = Delta * (u - z) rounded once to fp16 before the MMA (so
 * |w_hat| must stay below 65504).  Larger M (prefill) runs as consecutive
 * chunks of 256 tokens, each chunk as above, on the same workspace.  x is the activation already divided by the AWQ scale s.
 * Accuracy: |y - y_ref| <= 2e-3 * sum_k |x[m][k] * w_hat[n][k]| + 1e-3 per element,
 * y_ref the exact product with the dequantized weight.  y is the same on every
 * call, bit for bit, on every path: the split-K CUDA-core GEMV (M = 1..4 when
 * the whole-row kernels do not apply: K / 128 odd, or activations too large
 * to stage) adds at most two partial sums per output onto zero, and the
 * tensor-core path adds its partial tiles in a fixed order.
 *
 *   x        fp16 [M][K], device.     y  fp16 [M][N], device (output).
 *   qweight, scales, zeros as produced by awq_quantize_pack (layout v1).
 *   M, N >= 1;  K a multiple of group;  group == 128;  N*K, M*K, M*N below 2^31.
 *   workspace  device memory of at least w4a16_gemm_workspace_size(M, N, K, group)
 *              bytes, 16-byte aligned, ZERO-FILLED before its first use.  Every
 *              call that completes leaves the part that must start at zero (the
 *              first w4a16_gemm_workspace_size(min(M, 4), N, K, group) bytes)
 *              zero-filled again, so it can be reused by later calls on the same
 *              stream; the rest is scratch.  Calls that may run concurrently
 *              need distinct workspaces.  After W4A16_ERR_DEVICE it must be zero-filled
 *              again by the caller.
 */
W4A16_API w4a16_status w4a16_gemm(const void* x, const uint32_t* qweight, const void* scales,
                        const void* zeros, int M, int N, int K, int group, void* y,
                        void* workspace, size_t workspace_bytes, w4a16_stream_t stream);

/*
 * awq_search_workspace_size -- bytes of workspace that awq_search_alpha needs
 * on the current device for these sizes; 0 for invalid sizes.
 */
W4A16_API size_t awq_search_workspace_size(int N, int K, int T, int n_alpha, int group);

/*
 * awq_search_alpha -- the AWQ scaling-strength search over a caller's grid.
 *
 *   for each alpha = alphas[a]:
 *     s          = awq_act_scale(X, alpha)                   (fp16 [K])
 *     qweight, scales, zeros = awq_quantize_pack(W, s, group, bits, mode)
 *     x'         = fp16(X / s)                               (per element, one rounding)
 *     y_q        = w4a16_gemm(x', qweight, scales, zeros)    (fp16 [T][N])
 *     losses[a]  = mean over the T x N outputs of (y_q - y)^2,   y = X W^T
 *   *best = the first a with the smallest loss
 *
 * The objective is the AWQ one: the error of the layer's output with the
 * scaled, quantized weight and the divided activation against the unquantized
 * output, minimised over alpha by a grid search on calibration tokens
 * ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide, §AWQ,
 * slide 28; "Learning-ML-DL ch. 11", §11.4).  Every step for an alpha is the
 * library's own entry point above, so the codes of the chosen alpha are the
 * ones awq_quantize_pack produces for it.  y is formed once, in fp32 on the
 * CUDA cores, from the exact fp16 products; each loss is an fp64 sum in a fixed
 * order, so the losses repeat exactly from call to call, as the GEMM outputs do.
 *
 *   W        fp16 [N][K], device.    X  fp16 [T][K] calibration tokens, device.
 *   alphas   double [n_alpha], host, finite (the pages search [0, 1]).
 *   losses   double [n_alpha], host (output).   best  int, host (output), or NULL.
 *   N >= 1;  1 <= T <= 2^20;  K a multiple of group;  group == 128;  bits in {3, 4};
 *   1 <= n_alpha <= 4096;  N*K, T*K and T*N below 2^31.
 *   workspace  device memory of at least awq_search_workspace_size(N, K, T,
 *              n_alpha, group) bytes, 16-byte aligned, any contents; it is
 *              scratch (the call zero-fills what needs it).
 * Unlike the other calls this one is synchronous: it enqueues the work on
 * `stream`, waits for it and returns the losses.  W * s must stay finite in
 * fp16 for every alpha of the grid (see awq_quantize_pack).  Returns
 * W4A16_ERR_DEVICE if a GEMM kernel gave up waiting (losses then unspecified).
 */
W4A16_API w4a16_status awq_search_alpha(const void* W, const void* X, int N, int K, int T,
                                        const double* alphas, int n_alpha, int group, int bits,
                                        w4a16_mode mode, double* losses, int* best, void* workspace,
                                        size_t workspace_bytes, w4a16_stream_t stream);

/*
 * awq_reference_product -- the target of the search above, y = X W^T, on its own.
 *   X  fp16 [T][K], W fp16 [N][K], Y fp32 [T][N] (all device, 16-byte aligned).
 * Each output is the fp32 sum, in k order, of the exact fp16 x fp16 products:
 * the same kernel and order awq_search_alpha uses, offered so that a caller
 * can check or reuse the search's target.  Asynchronous on `stream`.
 *   N, K >= 1;  1 <= T <= 2^20;  N*K, T*K and T*N below 2^31.
 */
W4A16_API w4a16_status awq_reference_product(const void* X, const void* W, int T, int N, int K, float* Y,
                                             w4a16_stream_t stream);

/*
 * gptq_hessian -- the damped Hessian of GPTQ's layer objective.
 *
 *   H = 2 X^T X + lambda I,   lambda = damp * (sum_i (2 X^T X)[i][i]) / K
 *
 * ("CMU 11-868 LLM Systems: Model Quantization" reading guide, §L20 "GPTQ",
 * step 1: (2 X X^T + lambda I) with tokens as the columns of X; "Learning-ML-DL
 * ch. 11", §11.4: damping by a fraction of the mean diagonal, 0.01 in its
 * example.)  Entries are fp64 sums of the exact fp16 products in token order.
 *
 *   X  fp16 [T][K] calibration tokens, device.   H  fp64 [K][K], device (output).
 *   T, K >= 1;  K <= 32768;  T*K below 2^31;  damp finite and >= 0.
 */
W4A16_API w4a16_status gptq_hessian(const void* X, int T, int K, double damp, double* H,
                                    w4a16_stream_t stream);

/* gptq_sweep_workspace_size -- bytes of workspace gptq_sweep needs; 0 for invalid sizes. */
W4A16_API size_t gptq_sweep_workspace_size(int N, int K, int group);

/*
 * gptq_sweep -- GPTQ's error-compensating column sweep, emitting layout v1.
 *
 * Columns are quantized left to right in blocks of `group` columns, one block
 * per quantization group (§L20 "GPTQ": one column block at a time, a fixed
 * order; the error of each column, divided by G's diagonal element, updates
 * the rest of the block, then every column right of the block at once):
 *   at a block's first column: Delta, z from the block as it stands, by the
 *     formulas of awq_quantize_pack (ASYM: fp16((max - min) / (2^bits - 1)) and
 *     clamp(Round(-min / Delta)); SYM: fp16(max|w| / 2^(bits-1)) and 2^(bits-1));
 *   column i: u = clamp(Round(w / Delta) + z, 0, 2^bits - 1),
 *             e = (w - (u - z) Delta) / G[i][i];
 *   later columns j of the block: w_j -= e G[i][j];
 *   after the block, columns j right of it: w_j -= sum over the block's
 *     columns i, in order, of e_i G[i][j].
 * All arithmetic is fp64, one rounding per operation in that order, so the
 * result is identical on every call and bit-exact to that definition.
 *
 *   W        fp16 [N][K], device.
 *   G        fp64 [K][K], device: the upper-triangular factor with
 *            H^-1 = G^T G (G = Cholesky(H^-1)^T, §L20 step 1), positive diagonal.
 *   qweight  uint32 [N][K/8], scales, zeros  fp16 [N][K/group] (outputs, the
 *            format of awq_quantize_pack, for w4a16_gemm).
 *   N >= 1;  K a multiple of group, at most 32768;  group == 128;  bits in {3, 4}.
 *   workspace  at least gptq_sweep_workspace_size(N, K, group) bytes, any
 *              contents (an fp64 copy of W, the codes and one block of errors).
 * Asynchronous on `stream`.  G comes from gptq_factor (or the caller).
 */
W4A16_API w4a16_status gptq_sweep(const void* W, const double* G, int N, int K, int group, int bits,
                                  w4a16_mode mode, uint32_t* qweight, void* scales, void* zeros,
                                  void* workspace, size_t workspace_bytes, w4a16_stream_t stream);

/* gptq_factor_workspace_size -- bytes of workspace gptq_factor needs (2 K^2 fp64); 0 for invalid K. */
W4A16_API size_t gptq_factor_workspace_size(int K);

/*
 * gptq_factor -- G = Cholesky(H^-1)^T, the upper-triangular factor with
 * H^-1 = G^T G and a positive diagonal ([CMU] §L20 "GPTQ", step 1).
 *
 * With P the reversal of the index order, P H P = L L^T (Cholesky, left-looking,
 * fp64), and G = P L^-1 P (triangular inverse by forward substitution, fp64):
 * U = P L P is upper triangular with H = U U^T, so G = U^-1 satisfies
 * G^T G = H^-1 and, being upper triangular with a positive diagonal, is that
 * factor.  The sums run over warp lanes: G agrees with other implementations
 * to rounding (about 1e-12 relative at K = 4096), not bit for bit.  The call
 * enqueues 2K + 2 kernel launches (offline use).
 *
 *   H  fp64 [K][K] symmetric positive definite, device (gptq_hessian's output).
 *   G  fp64 [K][K], device (output; the lower triangle is written as zeros).
 *   1 <= K <= 32768;  workspace  gptq_factor_workspace_size(K) bytes, any contents.
 */
W4A16_API w4a16_status gptq_factor(const double* H, int K, double* G, void* workspace,
                                   size_t workspace_bytes, w4a16_stream_t stream);

/* gptq_quantize_workspace_size -- bytes of workspace gptq_quantize needs; 0 for invalid sizes. */
W4A16_API size_t gptq_quantize_workspace_size(int N, int K, int group);

/*
 * gptq_quantize -- GPTQ end to end: gptq_hessian(X, damp), gptq_factor, then
 * gptq_sweep(W, G), all on `stream`, into qweight / scales / zeros (layout v1,
 * the format w4a16_gemm reads).  Arguments as for those calls; T is the number
 * of calibration tokens in X (fp16 [T][K]).  The workspace (any contents) holds
 * H, G and the scratch of the factor and of the sweep.
 */
W4A16_API w4a16_status gptq_quantize(const void* W, const void* X, int N, int K, int T, double damp,
                                     int group, int bits, w4a16_mode mode, uint32_t* qweight,
                                     void* scales, void* zeros, void* workspace,
                                     size_t workspace_bytes, w4a16_stream_t stream);

/*
 * ---- W4A8 with progressive group quantization ------------------------------
 * "MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide, §QServe
 * (slides 47-57): 4-bit weights whose group scale is applied before the zero
 * point, so that the dequantized weight is an int8 value; 8-bit per-token
 * activations; int8 tensor cores; the conversion to floating point at the end.
 * The pages give no formulas; the readings these calls implement:
 *   level 1, per output channel n: s1[n] = fp16(max_k |W[n][k]| / 119)
 *     (fp16(1/119) for a zero row), w8 = clip(Round(W / s1), -119, 119);
 *   level 2, per group of 128 inputs: mx = max(max w8, 0), mn = min(min w8, 0),
 *     s2 = max(1, ceil((mx - mn) / 15)), z2 = clip(Round(-mn / s2), 0, 15),
 *     u = clip(Round(w8 / s2) + z2, 0, 15); zs = z2 * s2 (<= 240);
 *   the dequantized weight is w8_hat = u * s2 - zs (always within int8);
 *   activations, per token m: s_x[m] = fp16(max_k |x[m][k]| / 127) (fp16(1/127)
 *     for a zero token), x8 = clip(Round(x / s_x), -127, 127);
 *   acc[m][n] = sum_k x8[m][k] * w8_hat[n][k] exactly (int32),
 *   y[m][n] = fp16((acc * s_x[m]) * s1[n]), each product in fp64, one rounding.
 * Round is half-to-even; every quotient decides its integer exactly.  119 is
 * the largest level-1 range for which no w8_hat leaves int8.
 */

/*
 * w4a8_quantize_weight -- the two-level quantization above.
 *   W        fp16 [N][K], row-major (device).
 *   qweight  u32 [N][K/8] layout v1 codes (device, written).
 *   s1       fp16 [N];  s2, zs  uint8 [N][K/group] (device, written).
 * group == 128; K a multiple of 128, at most 65536.  Asynchronous on `stream`.
 */
W4A16_API w4a16_status w4a8_quantize_weight(const void* W, int N, int K, int group, uint32_t* qweight,
                                            void* s1, uint8_t* s2, uint8_t* zs, w4a16_stream_t stream);

/*
 * w4a8_quantize_act -- per-token int8 activations.
 *   x   fp16 [M][K] (device);  x8  int8 [M][K] (device, written);  sx  fp16 [M] (device, written).
 * 1 <= M <= 65535.  Asynchronous on `stream`.
 */
W4A16_API w4a16_status w4a8_quantize_act(const void* x, int M, int K, int8_t* x8, void* sx,
                                         w4a16_stream_t stream);

/* Workspace bytes w4a8_gemm needs (0 for invalid sizes); same layout rules as w4a16_gemm's. */
W4A16_API size_t w4a8_gemm_workspace_size(int M, int N, int K, int group);

/*
 * w4a8_gemm -- y = fp16((acc * s_x) * s1) with acc = x8 . w8_hat^T exact.
 *   x8 int8 [M][K], sx fp16 [M] (w4a8_quantize_act);  qweight, s1, s2, zs
 *   (w4a8_quantize_weight);  y fp16 [M][N] (written);  acc int32 [M][N] or NULL
 *   (written when given: the exact accumulators).  All device pointers,
 *   16-byte aligned.
 * M = 1..4 runs on CUDA cores (dp4a, the zero point taken out once per group);
 * larger M on the int8 tensor cores (tcgen05.mma kind::i8, w8_hat formed in
 * registers: one multiply by s2 per four codes and a bytewise subtraction of
 * zs), in chunks of 256 tokens.  Integer sums make y independent of the order
 * of addition.  The workspace (w4a8_gemm_workspace_size bytes) follows the
 * rules of w4a16_gemm's: zero-filled once by the caller, left so by each call.
 * Errors as w4a16_gemm; w4a16_gemm_check reports wait timeouts.
 */
W4A16_API w4a16_status w4a8_gemm(const int8_t* x8, const void* sx, const uint32_t* qweight, const void* s1,
                                 const uint8_t* s2, const uint8_t* zs, int M, int N, int K, int group, void* y,
                                 int32_t* acc, void* workspace, size_t workspace_bytes,
                                 w4a16_stream_t stream);

/*
 * w4a16_gemm_check -- synchronizes `stream` and reads the workspace's device
 * status word.  Returns W4A16_ERR_DEVICE if any earlier w4a16_gemm with this
 * workspace gave up waiting for its weight tiles (bounded waits, about 2 s),
 * W4A16_ERR_CUDA if the stream reports an error, else W4A16_OK.  The status word is
 * cleared by this call.
 */
W4A16_API w4a16_status w4a16_gemm_check(void* workspace, w4a16_stream_t stream);

/*
 * w4a16_wait_timeout_selftest -- diagnostics for the bounded waits behind
 * W4A16_ERR_DEVICE.  Launches one small kernel on `stream` that waits on a
 * shared-memory barrier nothing will ever complete, gives up after
 * `limit_us` microseconds (1 .. 1000000), and records the timeout in the
 * workspace's status word exactly as the GEMM kernels do.  A following
 * w4a16_gemm_check on the same workspace then returns W4A16_ERR_DEVICE.
 * Nothing faults or hangs: the wait is bounded by the device clock.
 *   workspace  at least 16 bytes, 16-byte aligned (a w4a16_gemm workspace).
 * Returns W4A16_ERR_ARG for a null workspace or a limit out of range,
 * W4A16_ERR_CUDA if the launch fails.
 */
W4A16_API w4a16_status w4a16_wait_timeout_selftest(void* workspace, int limit_us, w4a16_stream_t stream);

/*
 * w4a16_gemv_noalloc -- the split-K CUDA-core GEMV of w4a16_gemm (1 <= M <= 4)
 * for callers that cannot allocate device memory: inference servers that
 * reserve every buffer at start-up, plug-ins handed only the tensors they work
 * on, and hosts linking this library without a device allocator.  The pages
 * have no counterpart; it exists for those callers only.
 *
 * Instead of a caller workspace it uses a scratch array of
 * w4a16_gemv_noalloc_max_scratch() bytes (512 KiB) that is part of this
 * library's device data: every GPU that loads the library holds it until the
 * process exits.  The scratch needed is that of w4a16_gemm_workspace_size;
 * larger M * N is rejected with W4A16_ERR_SHAPE and a message.  The call
 * allocates nothing.  Its first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current) and caches it;
 * make that first call before any stream capture.  Each call clears the part
 * of the array it uses with an asynchronous memset on `stream`.  All calls
 * share the one array, so calls whose work may overlap on the GPU (streams
 * without ordering between them) race and must not be made.
 * Arguments, layouts and accuracy are those of w4a16_gemm.
 */
W4A16_API w4a16_status w4a16_gemv_noalloc(const void* x, const uint32_t* qweight, const void* scales,
                                          const void* zeros, int M, int N, int K, int group, void* y,
                                          w4a16_stream_t stream);

/* Size in bytes of the fixed scratch array used by w4a16_gemv_noalloc. */
W4A16_API size_t w4a16_gemv_noalloc_max_scratch(void);

/*
 * w4a16_gemv_noalloc_check -- the w4a16_gemm_check of the allocation-free GEMV
 * (the pages have no counterpart).  Synchronizes `stream`, reads the status
 * word of the current device's scratch array and clears it.  Returns
 * W4A16_ERR_DEVICE if a w4a16_gemv_noalloc kernel since the last call gave up
 * waiting for its weight tiles (its y is then incomplete), W4A16_ERR_CUDA if
 * the stream reports an error, else W4A16_OK.  Every w4a16_gemv_noalloc call
 * clears the status word when it starts, so check after a call and before the
 * next one.  Allocates nothing.
 */
W4A16_API w4a16_status w4a16_gemv_noalloc_check(w4a16_stream_t stream);

/*
 * w4a16_gemv_noalloc_timeout_selftest -- w4a16_wait_timeout_selftest aimed at
 * the scratch array's status word: one small kernel on `stream` waits on a
 * barrier nothing completes, gives up after `limit_us` microseconds
 * (1 .. 1000000) and records the timeout, so that w4a16_gemv_noalloc_check
 * then returns W4A16_ERR_DEVICE.  Nothing faults or hangs.  Returns
 * W4A16_ERR_ARG for a limit out of range, W4A16_ERR_CUDA if the launch fails.
 */
W4A16_API w4a16_status w4a16_gemv_noalloc_timeout_selftest(int limit_us, w4a16_stream_t stream);

/* Message for the last error on this thread ("" if none). */
W4A16_API const char* w4a16_last_error(void);

/* Packed layout version: 1 (see above). */
W4A16_API int w4a16_layout_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H_ */
