// w4a16_gemv_noalloc: the split-K CUDA-core GEMV of w4a16_gemm, for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc, or cannot call it at the moment they
// run a GEMV: code that runs under a fixed, pre-reserved memory budget (an
// inference server that sizes all of its buffers at start-up), plug-ins that
// receive only the tensors they work on and have no allocator of their own,
// and C or foreign-language hosts that link this library without a device
// allocator.  For them this entry point takes its scratch space (split-K fp32
// partial sums, row-block counters, a status word) from a fixed array that
// lives in this library's device data instead of a caller-provided workspace.
//
// The array is a file-scope __device__ variable of kNoallocScratchBytes
// bytes; every GPU that loads the library holds it until the process exits.
// Host code cannot use its name as a device address: the address is looked up
// once per device with cudaGetSymbolAddress (on the first call made while that
// device is current) and then cached.  Every call shares the one array and it
// keeps the previous call's contents, so each call first clears the part it
// uses (an asynchronous memset on the caller's stream).  Calls whose kernels
// may overlap on the GPU (different streams without ordering between them)
// race on the array and must not be made.
#include <cstdio>
#include <mutex>

#include "../../include/w4a16.h"
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr size_t kNoallocScratchBytes = 512 * 1024;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

w4a16_status noalloc_fail(w4a16_status st, const char* msg) {
  set_last_error(msg);
  return st;
}

// Device address of the scratch array on the current device, looked up on the
// first use and cached; null (with the message set) on failure.
void* scratch_base(const char* who) {
  char buf[160];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    snprintf(buf, sizeof(buf), "%s: no usable current device", who);
    set_last_error(buf);
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(buf, sizeof(buf), "%s: cudaGetSymbolAddress failed", who);
      set_last_error(buf);
      return nullptr;
    }
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace w4a16

using namespace w4a16;

extern "C" {

W4A16_API size_t w4a16_gemv_noalloc_max_scratch(void) { return kNoallocScratchBytes; }

W4A16_API w4a16_status w4a16_gemv_noalloc(const void* x, const uint32_t* qweight, const void* scales,
                                          const void* zeros, int M, int N, int K, int group, void* y,
                                          w4a16_stream_t stream) {
  set_last_error("");
  if (!x || !qweight || !scales || !zeros || !y) return noalloc_fail(W4A16_ERR_ARG, "w4a16_gemv_noalloc: null pointer");
  if (M < 1 || N < 1 || K < 1) return noalloc_fail(W4A16_ERR_ARG, "w4a16_gemv_noalloc: sizes must be >= 1");
  if (group != kGroup) return noalloc_fail(W4A16_ERR_UNSUPPORTED, "w4a16_gemv_noalloc: group must be 128");
  if (K % group) return noalloc_fail(W4A16_ERR_SHAPE, "w4a16_gemv_noalloc: K must be a multiple of the group");
  if (M > kMaxGemvM) return noalloc_fail(W4A16_ERR_UNSUPPORTED, "w4a16_gemv_noalloc: M must be at most 4");
  if (static_cast<long long>(N) * K >= (1ll << 31))
    return noalloc_fail(W4A16_ERR_SHAPE, "w4a16_gemv_noalloc: N*K too large");
  const uintptr_t mis = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(qweight) |
                        reinterpret_cast<uintptr_t>(scales) | reinterpret_cast<uintptr_t>(zeros) |
                        reinterpret_cast<uintptr_t>(y);
  if (mis & 15u) return noalloc_fail(W4A16_ERR_ALIGN, "w4a16_gemv_noalloc: pointers must be 16-byte aligned");
  const size_t need = workspace_bytes(M, N, K);
  if (need > kNoallocScratchBytes) {
    char buf[200];
    snprintf(buf, sizeof(buf),
             "w4a16_gemv_noalloc: M=%d N=%d needs %zu bytes of scratch, more than the fixed %zu", M, N, need,
             kNoallocScratchBytes);
    return noalloc_fail(W4A16_ERR_SHAPE, buf);
  }

  // device address of the scratch array on the current device (looked up once)
  void* base = scratch_base("w4a16_gemv_noalloc");
  if (!base) return W4A16_ERR_CUDA;

  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the kernel expects zeroed partial sums, counters and status word
  if (cudaMemsetAsync(base, 0, need, st) != cudaSuccess)
    return noalloc_fail(W4A16_ERR_CUDA, "w4a16_gemv_noalloc: clearing the scratch array failed");
  GemmProblem p{static_cast<const __half*>(x), qweight, static_cast<const __half*>(scales),
                static_cast<const __half*>(zeros), static_cast<__half*>(y), M, N, K};
  const cudaError_t e = launch_gemv(p, carve_workspace(base, M, N, K), st);
  if (e != cudaSuccess) return noalloc_fail(W4A16_ERR_CUDA, "w4a16_gemv_noalloc: kernel launch failed");
  return W4A16_OK;
}

W4A16_API w4a16_status w4a16_gemv_noalloc_check(w4a16_stream_t stream) {
  set_last_error("");
  void* base = scratch_base("w4a16_gemv_noalloc_check");
  if (!base) return W4A16_ERR_CUDA;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess)
    return noalloc_fail(W4A16_ERR_CUDA, "w4a16_gemv_noalloc_check: the stream reports an error");
  // the status word is the first word of the array (carve_workspace)
  uint32_t flag = 0;
  if (cudaMemcpy(&flag, base, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess)
    return noalloc_fail(W4A16_ERR_CUDA, "w4a16_gemv_noalloc_check: reading the status word failed");
  if (flag != kDevOk) {
    const uint32_t zero = 0;
    if (cudaMemcpy(base, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return noalloc_fail(W4A16_ERR_CUDA, "w4a16_gemv_noalloc_check: clearing the status word failed");
    return noalloc_fail(W4A16_ERR_DEVICE, "w4a16_gemv_noalloc: a kernel gave up waiting for its weight tiles");
  }
  return W4A16_OK;
}

W4A16_API w4a16_status w4a16_gemv_noalloc_timeout_selftest(int limit_us, w4a16_stream_t stream) {
  set_last_error("");
  if (limit_us < 1 || limit_us > 1000000)
    return noalloc_fail(W4A16_ERR_ARG, "w4a16_gemv_noalloc_timeout_selftest: limit_us must be 1 .. 1000000");
  void* base = scratch_base("w4a16_gemv_noalloc_timeout_selftest");
  if (!base) return W4A16_ERR_CUDA;
  if (launch_wait_timeout_probe(static_cast<uint32_t*>(base), static_cast<uint64_t>(limit_us) * 1000ull,
                                reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return noalloc_fail(W4A16_ERR_CUDA, "w4a16_gemv_noalloc_timeout_selftest: launch failed");
  return W4A16_OK;
}

}  // extern "C"
