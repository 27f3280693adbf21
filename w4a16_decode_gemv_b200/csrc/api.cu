// C ABI of the w4a16 library: argument checks, error reporting, dispatch.
// The operations themselves are specified in include/w4a16.h.
#include <atomic>
#include <vector>
#include <mutex>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <string>

#include "../../include/w4a16.h"
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

thread_local std::string g_last_error;

w4a16_status fail(w4a16_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
w4a16_status fail(w4a16_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

w4a16_status ok() {
  g_last_error.clear();
  return W4A16_OK;
}

w4a16_status cuda_fail(cudaError_t e, const char* what) {
  return fail(W4A16_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr long long kMaxElems = 1ll << 31;  // index arithmetic stays in 64 bits; sizes stay sane

}  // namespace

void set_last_error(const char* msg) { g_last_error = msg; }

int device_sm_count() {
  // per-device cache; threads that race on a first call store the same value
  static std::atomic<int> cached[128];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

cudaError_t ensure_func_attr(const void* func, cudaFuncAttribute attr, int value) {
  struct Entry {
    const void* func;
    int dev;
    cudaFuncAttribute attr;
    int value;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& en : done)
      if (en.func == func && en.dev == dev && en.attr == attr && en.value == value) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(func, attr, value);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    done.push_back({func, dev, attr, value});
  }
  return e;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("W4A16_NO_PDL");
    return !(v && v[0]);
  }();
  return on;
}

static size_t counter_bytes(int N) {
  const size_t row_blocks = (static_cast<size_t>(N) + 3) / 4;
  return (row_blocks * 4 + 15) / 16 * 16;
}

// Room for the CUDA-core GEMV partial sums (M x N fp32, at most kMaxGemvM rows).
static size_t gemv_acc_bytes(int M, int N) {
  const size_t m = static_cast<size_t>(M < kMaxGemvM ? M : kMaxGemvM);
  return (m * N * 4 + 15) / 16 * 16;
}

size_t workspace_bytes(int M, int N, int K) {
  (void)K;
  const size_t head = 16 + kFlagBytes + counter_bytes(N);
  if (M <= kMaxGemvM) return head + static_cast<size_t>(M) * N * 4;
  return head + gemv_acc_bytes(kMaxGemvM, N) + tc_partial_bytes(M);
}

Workspace carve_workspace(void* base, int M, int N, int K) {
  (void)K;
  uint8_t* p = static_cast<uint8_t*>(base);
  const size_t head = 16 + kFlagBytes + counter_bytes(N);
  Workspace w;
  w.status = reinterpret_cast<uint32_t*>(p);
  w.flags = reinterpret_cast<uint32_t*>(p + 16);
  w.counters = reinterpret_cast<uint32_t*>(p + 16 + kFlagBytes);
  w.acc = reinterpret_cast<float*>(p + head);
  w.part = M <= kMaxGemvM ? nullptr : reinterpret_cast<float*>(p + head + gemv_acc_bytes(kMaxGemvM, N));
  return w;
}

// The kernels for an M x N x K problem with M <= kMaxM: M = 1 on whole rows when
// the activation fits the kernel's staging; M = 2..8 on whole rows with
// register-sourced MMAs when K is a multiple of 256 and the activations fit,
// else M = 2..4 on whole rows or split-K on the CUDA cores; the rest (up to 256
// tokens) on the tcgen05 tensor cores.
static cudaError_t dispatch_gemm(const GemmProblem& p, const Workspace& ws, cudaStream_t st) {
  if (p.M == 1 && gemv_m1_supports(p.N, p.K)) return launch_gemv_m1(p, ws.status, st);
  if (gemv_mma_supports(p.M, p.N, p.K)) return launch_gemv_mma(p, ws.status, st);
  if (gemv_mt_supports(p.M, p.N, p.K)) return launch_gemv_mt(p, ws.status, st);
  if (p.M <= kMaxGemvM && gemv_supports(p.M, p.K)) return launch_gemv(p, ws, st);
  return launch_gemm_tc(p, ws, st);
}

cudaError_t gemm_chunks(const GemmProblem& p, void* workspace, cudaStream_t st) {
  // Chunk c starts kMaxM * c tokens in: its x and y offsets are multiples of
  // 512 bytes per input and per output channel, so both stay 16-byte aligned.
  // Stream order keeps the chunks' uses of the workspace apart (a chunk's
  // partial tiles and flags are touched only after its griddepcontrol.wait,
  // which waits for the previous chunk to complete).
  for (int t0 = 0; t0 < p.M; t0 += kMaxM) {
    GemmProblem c = p;
    c.M = p.M - t0 < kMaxM ? p.M - t0 : kMaxM;
    c.x = p.x + static_cast<size_t>(t0) * p.K;
    c.y = p.y + static_cast<size_t>(t0) * p.N;
    const cudaError_t e = dispatch_gemm(c, carve_workspace(workspace, c.M, p.N, p.K), st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Workspace of awq_search_alpha: every region starts on a 256-byte boundary.
struct SearchLayout {
  int gemm_rows;  // tokens of the GEMM workspace: min(T, kMaxM)
  size_t gemm, qweight, scales, zeros, s, xd, yq, yref, partial, sums, total;
};

static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

static SearchLayout search_layout(int N, int K, int T, int n_alpha) {
  SearchLayout L;
  L.gemm_rows = T < kMaxM ? T : kMaxM;
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  const size_t groups = static_cast<size_t>(N) * (K / kGroup);
  L.gemm = take(workspace_bytes(L.gemm_rows, N, K));
  L.qweight = take(static_cast<size_t>(N) * (K / 8) * 4);
  L.scales = take(groups * 2);
  L.zeros = take(groups * 2);
  L.s = take(static_cast<size_t>(K) * 2);
  L.xd = take(static_cast<size_t>(T) * K * 2);
  L.yq = take(static_cast<size_t>(T) * N * 2);
  L.yref = take(static_cast<size_t>(T) * N * 4);
  L.partial = take(static_cast<size_t>(n_alpha) * search_error_blocks() * 8);
  L.sums = take(static_cast<size_t>(n_alpha) * 8);
  L.total = off;
  return L;
}

constexpr int kMaxAlphas = 4096;
constexpr int kMaxW4A8K = 65536;  // |acc| < K * 127 * 127 stays below 2^31
constexpr int kMaxSearchTokens = 1 << 20;  // the target GEMM's grid holds T / 64 in its y dimension

}  // namespace w4a16

using namespace w4a16;

extern "C" {

const char* w4a16_last_error(void) { return g_last_error.c_str(); }

int w4a16_layout_version(void) { return 1; }

w4a16_status awq_act_scale(const void* X, int T, int K, double alpha, void* s, w4a16_stream_t stream) {
  if (!X || !s) return fail(W4A16_ERR_ARG, "awq_act_scale: null pointer");
  if (T < 1 || K < 1) return fail(W4A16_ERR_ARG, "awq_act_scale: T=%d K=%d must be >= 1", T, K);
  if (static_cast<long long>(T) * K >= kMaxElems) return fail(W4A16_ERR_SHAPE, "awq_act_scale: T*K too large");
  if (!std::isfinite(alpha)) return fail(W4A16_ERR_ARG, "awq_act_scale: alpha must be finite");
  if (!aligned16(X) || !aligned16(s)) return fail(W4A16_ERR_ALIGN, "awq_act_scale: pointers must be 16-byte aligned");
  cudaError_t e = launch_act_scale(static_cast<const __half*>(X), T, K, alpha, static_cast<__half*>(s),
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "awq_act_scale launch");
  return ok();
}

w4a16_status awq_quantize_pack(const void* W, const void* s, int N, int K, int group, int bits, w4a16_mode mode,
                               uint32_t* qweight, void* scales, void* zeros, w4a16_stream_t stream) {
  if (!W || !qweight || !scales || !zeros) return fail(W4A16_ERR_ARG, "awq_quantize_pack: null pointer");
  if (N < 1 || K < 1) return fail(W4A16_ERR_ARG, "awq_quantize_pack: N=%d K=%d must be >= 1", N, K);
  if (mode != W4A16_ASYM && mode != W4A16_SYM) return fail(W4A16_ERR_ARG, "awq_quantize_pack: bad mode %d", mode);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "awq_quantize_pack: group=%d (only 128)", group);
  if (bits != 3 && bits != 4) return fail(W4A16_ERR_UNSUPPORTED, "awq_quantize_pack: bits=%d (3 or 4)", bits);
  if (K % group) return fail(W4A16_ERR_SHAPE, "awq_quantize_pack: K=%d not a multiple of group=%d", K, group);
  if (static_cast<long long>(N) * K >= kMaxElems) return fail(W4A16_ERR_SHAPE, "awq_quantize_pack: N*K too large");
  if (!aligned16(W) || (s && !aligned16(s)) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros))
    return fail(W4A16_ERR_ALIGN, "awq_quantize_pack: pointers must be 16-byte aligned");
  cudaError_t e = launch_quantize_pack(static_cast<const __half*>(W), static_cast<const __half*>(s), N, K, bits,
                                       static_cast<int>(mode), qweight, static_cast<__half*>(scales),
                                       static_cast<__half*>(zeros), reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "awq_quantize_pack launch");
  return ok();
}

size_t w4a16_gemm_workspace_size(int M, int N, int K, int group) {
  if (M < 1 || N < 1 || K < 1 || group != kGroup || K % group) return 0;
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(M) * K >= kMaxElems ||
      static_cast<long long>(M) * N >= kMaxElems)
    return 0;
  return workspace_bytes(M < kMaxM ? M : kMaxM, N, K);
}

w4a16_status w4a16_gemm(const void* x, const uint32_t* qweight, const void* scales, const void* zeros, int M, int N,
                        int K, int group, void* y, void* workspace, size_t workspace_bytes_, w4a16_stream_t stream) {
  if (!x || !qweight || !scales || !zeros || !y) return fail(W4A16_ERR_ARG, "w4a16_gemm: null pointer");
  if (M < 1 || N < 1 || K < 1) return fail(W4A16_ERR_ARG, "w4a16_gemm: M=%d N=%d K=%d must be >= 1", M, N, K);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "w4a16_gemm: group=%d (only 128)", group);
  if (K % group) return fail(W4A16_ERR_SHAPE, "w4a16_gemm: K=%d not a multiple of group=%d", K, group);
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(M) * K >= kMaxElems ||
      static_cast<long long>(M) * N >= kMaxElems)
    return fail(W4A16_ERR_SHAPE, "w4a16_gemm: N*K, M*K or M*N too large");
  if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y))
    return fail(W4A16_ERR_ALIGN, "w4a16_gemm: pointers must be 16-byte aligned");
  const size_t need = workspace_bytes(M < kMaxM ? M : kMaxM, N, K);
  if (!workspace || workspace_bytes_ < need)
    return fail(W4A16_ERR_WORKSPACE, "w4a16_gemm: workspace of %zu bytes needed, %zu given", need, workspace_bytes_);
  if (!aligned16(workspace)) return fail(W4A16_ERR_ALIGN, "w4a16_gemm: workspace must be 16-byte aligned");
  GemmProblem p{static_cast<const __half*>(x), qweight, static_cast<const __half*>(scales),
                static_cast<const __half*>(zeros), static_cast<__half*>(y), M, N, K};
  const cudaError_t e = gemm_chunks(p, workspace, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return fail(W4A16_ERR_UNSUPPORTED, "w4a16_gemm: M=%d K=%d not supported yet", M, K);
  if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm launch");
  return ok();
}

size_t awq_search_workspace_size(int N, int K, int T, int n_alpha, int group) {
  if (N < 1 || K < 1 || T < 1 || T > kMaxSearchTokens || n_alpha < 1 || n_alpha > kMaxAlphas || group != kGroup ||
      K % group)
    return 0;
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(T) * K >= kMaxElems ||
      static_cast<long long>(T) * N >= kMaxElems)
    return 0;
  return search_layout(N, K, T, n_alpha).total;
}

w4a16_status awq_search_alpha(const void* W, const void* X, int N, int K, int T, const double* alphas, int n_alpha,
                              int group, int bits, w4a16_mode mode, double* losses, int* best, void* workspace,
                              size_t workspace_bytes_, w4a16_stream_t stream) {
  if (!W || !X || !alphas || !losses || !workspace) return fail(W4A16_ERR_ARG, "awq_search_alpha: null pointer");
  if (N < 1 || K < 1 || T < 1) return fail(W4A16_ERR_ARG, "awq_search_alpha: N=%d K=%d T=%d must be >= 1", N, K, T);
  if (T > kMaxSearchTokens) return fail(W4A16_ERR_SHAPE, "awq_search_alpha: T=%d (at most %d)", T, kMaxSearchTokens);
  if (n_alpha < 1 || n_alpha > kMaxAlphas)
    return fail(W4A16_ERR_ARG, "awq_search_alpha: n_alpha=%d (1 .. %d)", n_alpha, kMaxAlphas);
  for (int a = 0; a < n_alpha; ++a)
    if (!std::isfinite(alphas[a])) return fail(W4A16_ERR_ARG, "awq_search_alpha: alphas[%d] is not finite", a);
  if (mode != W4A16_ASYM && mode != W4A16_SYM) return fail(W4A16_ERR_ARG, "awq_search_alpha: bad mode %d", mode);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "awq_search_alpha: group=%d (only 128)", group);
  if (bits != 3 && bits != 4) return fail(W4A16_ERR_UNSUPPORTED, "awq_search_alpha: bits=%d (3 or 4)", bits);
  if (K % group) return fail(W4A16_ERR_SHAPE, "awq_search_alpha: K=%d not a multiple of group=%d", K, group);
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(T) * K >= kMaxElems ||
      static_cast<long long>(T) * N >= kMaxElems)
    return fail(W4A16_ERR_SHAPE, "awq_search_alpha: N*K, T*K or T*N too large");
  if (!aligned16(W) || !aligned16(X) || !aligned16(workspace))
    return fail(W4A16_ERR_ALIGN, "awq_search_alpha: W, X and workspace must be 16-byte aligned");
  const SearchLayout L = search_layout(N, K, T, n_alpha);
  if (workspace_bytes_ < L.total)
    return fail(W4A16_ERR_WORKSPACE, "awq_search_alpha: workspace of %zu bytes needed, %zu given", L.total,
                workspace_bytes_);

  uint8_t* base = static_cast<uint8_t*>(workspace);
  const __half* Wh = static_cast<const __half*>(W);
  const __half* Xh = static_cast<const __half*>(X);
  uint32_t* qweight = reinterpret_cast<uint32_t*>(base + L.qweight);
  __half* scales = reinterpret_cast<__half*>(base + L.scales);
  __half* zeros = reinterpret_cast<__half*>(base + L.zeros);
  __half* s = reinterpret_cast<__half*>(base + L.s);
  __half* xd = reinterpret_cast<__half*>(base + L.xd);
  __half* yq = reinterpret_cast<__half*>(base + L.yq);
  float* yref = reinterpret_cast<float*>(base + L.yref);
  double* partial = reinterpret_cast<double*>(base + L.partial);
  double* sums = reinterpret_cast<double*>(base + L.sums);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int blocks = search_error_blocks();

  // The GEMM workspace must start zeroed; its status word doubles as the search's.
  cudaError_t e = cudaMemsetAsync(base + L.gemm, 0, workspace_bytes(L.gemm_rows, N, K), st);
  if (e != cudaSuccess) return cuda_fail(e, "awq_search_alpha: clear workspace");
  e = launch_reference_gemm(Xh, Wh, T, N, K, yref, st);
  if (e != cudaSuccess) return cuda_fail(e, "awq_search_alpha: reference product");
  for (int a = 0; a < n_alpha && e == cudaSuccess; ++a) {
    e = launch_act_scale(Xh, T, K, alphas[a], s, st);
    if (e == cudaSuccess)
      e = launch_quantize_pack(Wh, s, N, K, bits, static_cast<int>(mode), qweight, scales, zeros, st);
    if (e == cudaSuccess) e = launch_divide_activation(Xh, s, T, K, xd, st);
    if (e == cudaSuccess) e = gemm_chunks(GemmProblem{xd, qweight, scales, zeros, yq, T, N, K}, base + L.gemm, st);
    if (e == cudaSuccess)
      e = launch_squared_error(yq, yref, static_cast<long long>(T) * N, partial + static_cast<size_t>(a) * blocks, st);
  }
  if (e == cudaErrorNotSupported) return fail(W4A16_ERR_UNSUPPORTED, "awq_search_alpha: K=%d not supported", K);
  if (e != cudaSuccess) return cuda_fail(e, "awq_search_alpha launch");
  e = launch_sum_partials(partial, n_alpha, sums, st);
  if (e != cudaSuccess) return cuda_fail(e, "awq_search_alpha: loss sums");
  uint32_t flag = 0;
  e = cudaMemcpyAsync(losses, sums, static_cast<size_t>(n_alpha) * 8, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&flag, base + L.gemm, sizeof(flag), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "awq_search_alpha: read losses");
  if (flag != kDevOk)
    return fail(W4A16_ERR_DEVICE, "awq_search_alpha: a GEMM kernel gave up waiting for its weight tiles (status %u)",
                flag);
  const double count = static_cast<double>(T) * N;
  int arg = 0;
  for (int a = 0; a < n_alpha; ++a) {
    losses[a] /= count;
    if (losses[a] < losses[arg]) arg = a;
  }
  if (best) *best = arg;
  return ok();
}

w4a16_status awq_reference_product(const void* X, const void* W, int T, int N, int K, float* Y,
                                   w4a16_stream_t stream) {
  if (!X || !W || !Y) return fail(W4A16_ERR_ARG, "awq_reference_product: null pointer");
  if (N < 1 || K < 1 || T < 1) return fail(W4A16_ERR_ARG, "awq_reference_product: N=%d K=%d T=%d must be >= 1", N, K, T);
  if (T > kMaxSearchTokens) return fail(W4A16_ERR_SHAPE, "awq_reference_product: T=%d (at most %d)", T, kMaxSearchTokens);
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(T) * K >= kMaxElems ||
      static_cast<long long>(T) * N >= kMaxElems)
    return fail(W4A16_ERR_SHAPE, "awq_reference_product: N*K, T*K or T*N too large");
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y))
    return fail(W4A16_ERR_ALIGN, "awq_reference_product: pointers must be 16-byte aligned");
  const cudaError_t e = launch_reference_gemm(static_cast<const __half*>(X), static_cast<const __half*>(W), T, N, K, Y,
                                              reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "awq_reference_product launch");
  return ok();
}

w4a16_status gptq_hessian(const void* X, int T, int K, double damp, double* H, w4a16_stream_t stream) {
  if (!X || !H) return fail(W4A16_ERR_ARG, "gptq_hessian: null pointer");
  if (T < 1 || K < 1) return fail(W4A16_ERR_ARG, "gptq_hessian: T=%d K=%d must be >= 1", T, K);
  if (!std::isfinite(damp) || damp < 0) return fail(W4A16_ERR_ARG, "gptq_hessian: damp must be finite and >= 0");
  if (K > kMaxGptqK) return fail(W4A16_ERR_SHAPE, "gptq_hessian: K=%d (at most %d)", K, kMaxGptqK);
  if (static_cast<long long>(T) * K >= kMaxElems) return fail(W4A16_ERR_SHAPE, "gptq_hessian: T*K too large");
  if (!aligned16(X) || !aligned16(H)) return fail(W4A16_ERR_ALIGN, "gptq_hessian: pointers must be 16-byte aligned");
  const cudaError_t e = launch_gptq_hessian(static_cast<const __half*>(X), T, K, damp, H,
                                            reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gptq_hessian launch");
  return ok();
}

size_t gptq_sweep_workspace_size(int N, int K, int group) {
  if (N < 1 || K < 1 || group != kGroup || K % group || K > kMaxGptqK) return 0;
  if (static_cast<long long>(N) * K >= kMaxElems) return 0;
  return gptq_sweep_workspace_bytes(N, K);
}

w4a16_status gptq_sweep(const void* W, const double* G, int N, int K, int group, int bits, w4a16_mode mode,
                        uint32_t* qweight, void* scales, void* zeros, void* workspace, size_t workspace_bytes_,
                        w4a16_stream_t stream) {
  if (!W || !G || !qweight || !scales || !zeros || !workspace) return fail(W4A16_ERR_ARG, "gptq_sweep: null pointer");
  if (N < 1 || K < 1) return fail(W4A16_ERR_ARG, "gptq_sweep: N=%d K=%d must be >= 1", N, K);
  if (mode != W4A16_ASYM && mode != W4A16_SYM) return fail(W4A16_ERR_ARG, "gptq_sweep: bad mode %d", mode);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "gptq_sweep: group=%d (only 128)", group);
  if (bits != 3 && bits != 4) return fail(W4A16_ERR_UNSUPPORTED, "gptq_sweep: bits=%d (3 or 4)", bits);
  if (K % group) return fail(W4A16_ERR_SHAPE, "gptq_sweep: K=%d not a multiple of group=%d", K, group);
  if (K > kMaxGptqK) return fail(W4A16_ERR_SHAPE, "gptq_sweep: K=%d (at most %d)", K, kMaxGptqK);
  if (static_cast<long long>(N) * K >= kMaxElems) return fail(W4A16_ERR_SHAPE, "gptq_sweep: N*K too large");
  if (!aligned16(W) || !aligned16(G) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      !aligned16(workspace))
    return fail(W4A16_ERR_ALIGN, "gptq_sweep: pointers must be 16-byte aligned");
  const size_t need = gptq_sweep_workspace_bytes(N, K);
  if (workspace_bytes_ < need)
    return fail(W4A16_ERR_WORKSPACE, "gptq_sweep: workspace of %zu bytes needed, %zu given", need, workspace_bytes_);
  const cudaError_t e = launch_gptq_sweep(static_cast<const __half*>(W), G, N, K, bits, static_cast<int>(mode),
                                          qweight, static_cast<__half*>(scales), static_cast<__half*>(zeros),
                                          workspace, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gptq_sweep launch");
  return ok();
}

size_t gptq_factor_workspace_size(int K) {
  if (K < 1 || K > kMaxGptqK) return 0;
  return gptq_factor_workspace_bytes(K);
}

w4a16_status gptq_factor(const double* H, int K, double* G, void* workspace, size_t workspace_bytes_,
                         w4a16_stream_t stream) {
  if (!H || !G || !workspace) return fail(W4A16_ERR_ARG, "gptq_factor: null pointer");
  if (K < 1) return fail(W4A16_ERR_ARG, "gptq_factor: K=%d must be >= 1", K);
  if (K > kMaxGptqK) return fail(W4A16_ERR_SHAPE, "gptq_factor: K=%d (at most %d)", K, kMaxGptqK);
  if (!aligned16(H) || !aligned16(G) || !aligned16(workspace))
    return fail(W4A16_ERR_ALIGN, "gptq_factor: pointers must be 16-byte aligned");
  const size_t need = gptq_factor_workspace_bytes(K);
  if (workspace_bytes_ < need)
    return fail(W4A16_ERR_WORKSPACE, "gptq_factor: workspace of %zu bytes needed, %zu given", need, workspace_bytes_);
  const cudaError_t e = launch_gptq_factor(H, K, G, workspace, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "gptq_factor launch");
  return ok();
}

// gptq_quantize's workspace: H, G, the factor's scratch, the sweep's, each 256-byte aligned.
static size_t gptq_matrix_bytes(int K) { return (static_cast<size_t>(K) * K * 8 + 255) / 256 * 256; }

size_t gptq_quantize_workspace_size(int N, int K, int group) {
  if (gptq_sweep_workspace_size(N, K, group) == 0) return 0;
  return 2 * gptq_matrix_bytes(K) + gptq_factor_workspace_bytes(K) + gptq_sweep_workspace_bytes(N, K);
}

w4a16_status gptq_quantize(const void* W, const void* X, int N, int K, int T, double damp, int group, int bits,
                           w4a16_mode mode, uint32_t* qweight, void* scales, void* zeros, void* workspace,
                           size_t workspace_bytes_, w4a16_stream_t stream) {
  if (!W || !X || !qweight || !scales || !zeros || !workspace)
    return fail(W4A16_ERR_ARG, "gptq_quantize: null pointer");
  if (N < 1 || K < 1 || T < 1) return fail(W4A16_ERR_ARG, "gptq_quantize: N=%d K=%d T=%d must be >= 1", N, K, T);
  if (!std::isfinite(damp) || damp < 0) return fail(W4A16_ERR_ARG, "gptq_quantize: damp must be finite and >= 0");
  if (mode != W4A16_ASYM && mode != W4A16_SYM) return fail(W4A16_ERR_ARG, "gptq_quantize: bad mode %d", mode);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "gptq_quantize: group=%d (only 128)", group);
  if (bits != 3 && bits != 4) return fail(W4A16_ERR_UNSUPPORTED, "gptq_quantize: bits=%d (3 or 4)", bits);
  if (K % group) return fail(W4A16_ERR_SHAPE, "gptq_quantize: K=%d not a multiple of group=%d", K, group);
  if (K > kMaxGptqK) return fail(W4A16_ERR_SHAPE, "gptq_quantize: K=%d (at most %d)", K, kMaxGptqK);
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(T) * K >= kMaxElems)
    return fail(W4A16_ERR_SHAPE, "gptq_quantize: N*K or T*K too large");
  if (!aligned16(W) || !aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      !aligned16(workspace))
    return fail(W4A16_ERR_ALIGN, "gptq_quantize: pointers must be 16-byte aligned");
  const size_t need = gptq_quantize_workspace_size(N, K, group);
  if (workspace_bytes_ < need)
    return fail(W4A16_ERR_WORKSPACE, "gptq_quantize: workspace of %zu bytes needed, %zu given", need,
                workspace_bytes_);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  double* H = reinterpret_cast<double*>(base);
  double* G = reinterpret_cast<double*>(base + gptq_matrix_bytes(K));
  void* fws = base + 2 * gptq_matrix_bytes(K);
  void* sws = base + 2 * gptq_matrix_bytes(K) + gptq_factor_workspace_bytes(K);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_gptq_hessian(static_cast<const __half*>(X), T, K, damp, H, st);
  if (e == cudaSuccess) e = launch_gptq_factor(H, K, G, fws, st);
  if (e == cudaSuccess)
    e = launch_gptq_sweep(static_cast<const __half*>(W), G, N, K, bits, static_cast<int>(mode), qweight,
                          static_cast<__half*>(scales), static_cast<__half*>(zeros), sws, st);
  if (e != cudaSuccess) return cuda_fail(e, "gptq_quantize launch");
  return ok();
}

w4a16_status w4a8_quantize_weight(const void* W, int N, int K, int group, uint32_t* qweight, void* s1, uint8_t* s2,
                                  uint8_t* zs, w4a16_stream_t stream) {
  if (!W || !qweight || !s1 || !s2 || !zs) return fail(W4A16_ERR_ARG, "w4a8_quantize_weight: null pointer");
  if (N < 1 || K < 1) return fail(W4A16_ERR_ARG, "w4a8_quantize_weight: N=%d K=%d must be >= 1", N, K);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "w4a8_quantize_weight: group=%d (only 128)", group);
  if (K % group) return fail(W4A16_ERR_SHAPE, "w4a8_quantize_weight: K=%d not a multiple of group=%d", K, group);
  if (K > kMaxW4A8K) return fail(W4A16_ERR_SHAPE, "w4a8_quantize_weight: K=%d (at most %d)", K, kMaxW4A8K);
  if (static_cast<long long>(N) * K >= kMaxElems) return fail(W4A16_ERR_SHAPE, "w4a8_quantize_weight: N*K too large");
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(s1) || !aligned16(s2) || !aligned16(zs))
    return fail(W4A16_ERR_ALIGN, "w4a8_quantize_weight: pointers must be 16-byte aligned");
  const cudaError_t e = launch_w4a8_quantize_weight(static_cast<const __half*>(W), N, K, qweight,
                                                    static_cast<__half*>(s1), s2, zs,
                                                    reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "w4a8_quantize_weight launch");
  return ok();
}

w4a16_status w4a8_quantize_act(const void* x, int M, int K, int8_t* x8, void* sx, w4a16_stream_t stream) {
  if (!x || !x8 || !sx) return fail(W4A16_ERR_ARG, "w4a8_quantize_act: null pointer");
  if (M < 1 || K < 1) return fail(W4A16_ERR_ARG, "w4a8_quantize_act: M=%d K=%d must be >= 1", M, K);
  if (M > 65535) return fail(W4A16_ERR_SHAPE, "w4a8_quantize_act: M=%d (at most 65535)", M);
  if (static_cast<long long>(M) * K >= kMaxElems) return fail(W4A16_ERR_SHAPE, "w4a8_quantize_act: M*K too large");
  if (!aligned16(x) || !aligned16(x8) || !aligned16(sx))
    return fail(W4A16_ERR_ALIGN, "w4a8_quantize_act: pointers must be 16-byte aligned");
  const cudaError_t e = launch_w4a8_quantize_act(static_cast<const __half*>(x), M, K, x8, static_cast<__half*>(sx),
                                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "w4a8_quantize_act launch");
  return ok();
}

size_t w4a8_gemm_workspace_size(int M, int N, int K, int group) {
  if (M < 1 || N < 1 || K < 1 || group != kGroup || K % group || K > kMaxW4A8K) return 0;
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(M) * K >= kMaxElems ||
      static_cast<long long>(M) * N >= kMaxElems)
    return 0;
  return workspace_bytes(M < kMaxM ? M : kMaxM, N, K);
}

w4a16_status w4a8_gemm(const int8_t* x8, const void* sx, const uint32_t* qweight, const void* s1, const uint8_t* s2,
                       const uint8_t* zs, int M, int N, int K, int group, void* y, int32_t* acc, void* workspace,
                       size_t workspace_bytes_, w4a16_stream_t stream) {
  if (!x8 || !sx || !qweight || !s1 || !s2 || !zs || !y) return fail(W4A16_ERR_ARG, "w4a8_gemm: null pointer");
  if (M < 1 || N < 1 || K < 1) return fail(W4A16_ERR_ARG, "w4a8_gemm: M=%d N=%d K=%d must be >= 1", M, N, K);
  if (group != kGroup) return fail(W4A16_ERR_UNSUPPORTED, "w4a8_gemm: group=%d (only 128)", group);
  if (K % group) return fail(W4A16_ERR_SHAPE, "w4a8_gemm: K=%d not a multiple of group=%d", K, group);
  if (K > kMaxW4A8K) return fail(W4A16_ERR_SHAPE, "w4a8_gemm: K=%d (at most %d)", K, kMaxW4A8K);
  if (static_cast<long long>(N) * K >= kMaxElems || static_cast<long long>(M) * K >= kMaxElems ||
      static_cast<long long>(M) * N >= kMaxElems)
    return fail(W4A16_ERR_SHAPE, "w4a8_gemm: N*K, M*K or M*N too large");
  if (!aligned16(x8) || !aligned16(sx) || !aligned16(qweight) || !aligned16(s1) || !aligned16(s2) ||
      !aligned16(zs) || !aligned16(y) || (acc && !aligned16(acc)))
    return fail(W4A16_ERR_ALIGN, "w4a8_gemm: pointers must be 16-byte aligned");
  const size_t need = workspace_bytes(M < kMaxM ? M : kMaxM, N, K);
  if (!workspace || workspace_bytes_ < need)
    return fail(W4A16_ERR_WORKSPACE, "w4a8_gemm: workspace of %zu bytes needed, %zu given", need, workspace_bytes_);
  if (!aligned16(workspace)) return fail(W4A16_ERR_ALIGN, "w4a8_gemm: workspace must be 16-byte aligned");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  // chunks of kMaxM tokens: x8, s_x, y and acc offsets stay 16-byte aligned (kMaxM * 2 bytes per token of s_x)
  for (int t0 = 0; t0 < M && e == cudaSuccess; t0 += kMaxM) {
    W4A8Problem c{x8 + static_cast<size_t>(t0) * K, static_cast<const __half*>(sx) + t0, qweight,
                  static_cast<const __half*>(s1), s2, zs, static_cast<__half*>(y) + static_cast<size_t>(t0) * N,
                  acc ? acc + static_cast<size_t>(t0) * N : nullptr, M - t0 < kMaxM ? M - t0 : kMaxM, N, K};
    const Workspace ws = carve_workspace(workspace, c.M, N, K);
    if (w4a8_gemv_supports(c.M, N, K))
      e = launch_w4a8_gemv(c, ws.status, st);
    else
      e = launch_w4a8_gemm_tc(c, ws, st);
  }
  if (e == cudaErrorNotSupported) return fail(W4A16_ERR_UNSUPPORTED, "w4a8_gemm: M=%d N=%d K=%d not supported", M, N, K);
  if (e != cudaSuccess) return cuda_fail(e, "w4a8_gemm launch");
  return ok();
}

w4a16_status w4a16_wait_timeout_selftest(void* workspace, int limit_us, w4a16_stream_t stream) {
  if (!workspace || !aligned16(workspace))
    return fail(W4A16_ERR_ARG, "w4a16_wait_timeout_selftest: workspace must be non-null and 16-byte aligned");
  if (limit_us < 1 || limit_us > 1000000)
    return fail(W4A16_ERR_ARG, "w4a16_wait_timeout_selftest: limit_us=%d (1 .. 1000000)", limit_us);
  const cudaError_t e = launch_wait_timeout_probe(static_cast<uint32_t*>(workspace),
                                                  static_cast<uint64_t>(limit_us) * 1000ull,
                                                  reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "w4a16_wait_timeout_selftest launch");
  return ok();
}

w4a16_status w4a16_gemm_check(void* workspace, w4a16_stream_t stream) {
  if (!workspace) return fail(W4A16_ERR_ARG, "w4a16_gemm_check: null workspace");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm_check: stream");
  uint32_t flag = 0;
  e = cudaMemcpy(&flag, workspace, sizeof(flag), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm_check: read status");
  if (flag != kDevOk) {
    // a kernel that gave up may have left partial-tile flags set: clear them with the status word
    e = cudaMemset(workspace, 0, 16 + kFlagBytes);
    if (e != cudaSuccess) return cuda_fail(e, "w4a16_gemm_check: clear status");
    return fail(W4A16_ERR_DEVICE, "w4a16_gemm: a kernel gave up waiting for its weight tiles (status %u)", flag);
  }
  return ok();
}

}  // extern "C"
