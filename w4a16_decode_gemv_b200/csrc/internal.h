// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstddef>
#include <cstdint>

namespace w4a16 {

constexpr int kGroup = 128;        // group size along K (the only one supported)
constexpr int kMaxGemvM = 4;       // largest M the CUDA-core GEMV handles
constexpr int kMaxM = 256;         // largest M of one launch sequence; larger M runs in chunks of it
constexpr int kMaxFlags = 1024;    // partial-tile flags of the tensor-core path (one per CTA)

// Replaces the calling thread's message returned by w4a16_last_error().
void set_last_error(const char* msg);

// Streaming-multiprocessor count of the current device (cached per device).
int device_sm_count();

// cudaFuncSetAttribute(func, attr, value), called once per kernel, device,
// attribute and value: the attribute lives in the device's context, so later
// launches need not set it again (it costs a driver call).  Not safe across a
// cudaDeviceReset of the device, which discards the context's settings.
cudaError_t ensure_func_attr(const void* func, cudaFuncAttribute attr, int value);

// Whether the GEMV kernels are launched with programmatic dependent launch
// (on unless the environment variable W4A16_NO_PDL is set to a non-empty value).
bool pdl_enabled();

cudaError_t launch_act_scale(const __half* X, int T, int K, double alpha, __half* s, cudaStream_t st);

cudaError_t launch_quantize_pack(const __half* W, const __half* s, int N, int K, int bits, int mode,
                                 uint32_t* qweight, __half* scales, __half* zeros, cudaStream_t st);

// Workspace: [status word | padding to 16 B] [kMaxFlags partial-tile flags of
// the tensor-core path] [row-block counters, padded to 16 B] [fp32 partial sums
// M x N of the CUDA-core GEMV, M <= 4] and, for M >= 5, after room for 4 x N
// GEMV partials: the tensor-core path's partial tiles (one per CTA of 128 x MP
// fp32, MP the launch's token tile).  The flags, counters and GEMV partials must
// be zero when a kernel starts and are left zero; the partial tiles are
// scratch, written before they are read.
struct Workspace {
  uint32_t* status;
  uint32_t* flags;
  uint32_t* counters;
  float* acc;
  float* part;  // tensor-core partial tiles (M >= 5 only), after the GEMV region
};
constexpr size_t kFlagBytes = kMaxFlags * 4;
size_t workspace_bytes(int M, int N, int K);
Workspace carve_workspace(void* base, int M, int N, int K);

struct GemmProblem {
  const __half* x;
  const uint32_t* qweight;
  const __half* scales;
  const __half* zeros;
  __half* y;
  int M, N, K;
};

// The M = 1 decode GEMV (gemv_m1.cu): whole rows per CTA, no workspace.
bool gemv_m1_supports(int N, int K);
cudaError_t launch_gemv_m1(const GemmProblem& p, uint32_t* status, cudaStream_t st);

// The M = 2..8 GEMV on mma.sync (gemv_mma.cu): whole rows per CTA, no
// workspace; false when K is not a multiple of 256 or the staged activations of
// M tokens leave no room for two ring stages.
bool gemv_mma_supports(int M, int N, int K);
cudaError_t launch_gemv_mma(const GemmProblem& p, uint32_t* status, cudaStream_t st);

// The M = 2..4 GEMV (gemv_mt.cu): whole rows per CTA, no workspace; false when
// the staged activations of M tokens do not fit in shared memory.
bool gemv_mt_supports(int M, int N, int K);
cudaError_t launch_gemv_mt(const GemmProblem& p, uint32_t* status, cudaStream_t st);

// The split-K CUDA-core GEMV for small M (gemv.cu).
bool gemv_supports(int M, int K);
cudaError_t launch_gemv(const GemmProblem& p, const Workspace& ws, cudaStream_t st);

// The tensor-core GEMM (gemm_tc.cu), M = 5..256 per launch, and the bytes of
// its partial tiles on the current device.
size_t tc_partial_bytes(int M);
cudaError_t launch_gemm_tc(const GemmProblem& p, const Workspace& ws, cudaStream_t st);
// One CTA waits on a shared-memory barrier that nothing completes, gives up
// after limit_ns and sets kDevWaitTimeout in *status (the GEMM kernels' path).
cudaError_t launch_wait_timeout_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t st);

// The kernels w4a16_gemm runs for p (api.cu): one launch sequence per chunk of
// at most kMaxM tokens, all on the workspace at `workspace` (sized for
// min(M, kMaxM) tokens).
cudaError_t gemm_chunks(const GemmProblem& p, void* workspace, cudaStream_t st);

// Kernels of the AWQ alpha search (awq_search.cu).  Y = X W^T in fp32 (X [T][K],
// W [N][K] fp16); Xd = fp16(X / s); per-block fp64 partial sums of (Yq - Y)^2
// over `total` elements, search_error_blocks() of them; sums[a] = the n_alpha
// groups of partials added in block order.
int search_error_blocks();
cudaError_t launch_reference_gemm(const __half* X, const __half* W, int T, int N, int K, float* Y, cudaStream_t st);
cudaError_t launch_divide_activation(const __half* X, const __half* s, int T, int K, __half* Xd, cudaStream_t st);
cudaError_t launch_squared_error(const __half* Yq, const float* Y, long long total, double* partial, cudaStream_t st);
cudaError_t launch_sum_partials(const double* partial, int n_alpha, double* sums, cudaStream_t st);

// GPTQ (gptq.cu): H = 2 X^T X + damp * mean(diag) I in fp64 [K][K]; the column
// sweep with a given upper-triangular factor G, writing layout-v1 codes, Delta
// and z; the sweep's workspace: the fp64 working copy of W, the codes and one
// block of errors.
constexpr int kMaxGptqK = 32768;
cudaError_t launch_gptq_hessian(const __half* X, int T, int K, double damp, double* H, cudaStream_t st);
size_t gptq_sweep_workspace_bytes(int N, int K);
size_t gptq_factor_workspace_bytes(int K);
cudaError_t launch_gptq_factor(const double* H, int K, double* G, void* workspace, cudaStream_t st);
cudaError_t launch_gptq_sweep(const __half* W, const double* G, int N, int K, int bits, int mode, uint32_t* qweight,
                              __half* scales, __half* zeros, void* workspace, cudaStream_t st);

// W4A8 (w4a8_quant.cu, w4a8_gemv.cu, gemm_tc.cu): the weight and activation
// quantizers, and the product on CUDA cores (M <= 4) or tensor cores (int8 MMA).
struct W4A8Problem {
  const int8_t* x8;
  const __half* sx;
  const uint32_t* qweight;
  const __half* s1;
  const uint8_t* s2;
  const uint8_t* zs;
  __half* y;
  int32_t* acc;  // optional exact accumulators [M][N]
  int M, N, K;
};
cudaError_t launch_w4a8_quantize_weight(const __half* W, int N, int K, uint32_t* qweight, __half* s1, uint8_t* s2,
                                        uint8_t* zs, cudaStream_t st);
cudaError_t launch_w4a8_quantize_act(const __half* x, int M, int K, int8_t* x8, __half* sx, cudaStream_t st);
bool w4a8_gemv_supports(int M, int N, int K);
cudaError_t launch_w4a8_gemv(const W4A8Problem& p, uint32_t* status, cudaStream_t st);
cudaError_t launch_w4a8_gemm_tc(const W4A8Problem& p, const Workspace& ws, cudaStream_t st);

// cuTensorMapEncodeTiled through the runtime's driver entry point (null if absent).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace w4a16
