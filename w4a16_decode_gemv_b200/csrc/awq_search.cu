// Kernels of the AWQ scaling-strength search.
//
//   L(alpha) = mean over outputs of (Q(W s)(s^-1 X) - W X)^2,   s = s_X^alpha,
//   alpha*   = argmin over the caller's grid
//
// ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide, §AWQ,
// slide 28: the scale comes from the activation magnitude alone, and the search
// minimises the error of the layer's output, not of the weights; a small grid
// search on calibration data picks alpha.)  The search itself runs the
// library's own steps for every alpha -- awq_act_scale, awq_quantize_pack and
// the W4A16 GEMM -- and these kernels supply the rest: the target W X, once; the
// divided activation fp16(X / s); and the squared error of the quantized output
// against the target.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

// ---- the target Y = X W^T in fp32 ----------------------------------------------
// A tiled CUDA-core GEMM: a CTA computes a 64 (tokens) x 64 (outputs) tile,
// thread (ty, tx) a 4 x 4 block of it, over K in chunks of 32 staged in
// shared memory as fp32.  The fp16 products are exact in fp32 and every output
// adds them in k order, so the result is the same on every run.  It runs once
// per search; the W4A16 path under test does not use it.
constexpr int kRefTile = 64;
constexpr int kRefChunk = 32;

__global__ void __launch_bounds__(256) ref_gemm_kernel(const __half* __restrict__ X, const __half* __restrict__ W,
                                                       int T, int N, int K, float* __restrict__ Y) {
  __shared__ float xs[kRefChunk][kRefTile + 4];  // [k][t]
  __shared__ float ws[kRefChunk][kRefTile + 4];  // [k][n]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int t0 = blockIdx.y * kRefTile, n0 = blockIdx.x * kRefTile;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kRefChunk) {
    // 64 rows x 32 inputs of X and of W: 8 values of each per thread
    for (int e = threadIdx.x; e < kRefTile * kRefChunk; e += 256) {
      const int r = e / kRefChunk, c = e % kRefChunk;
      const int t = t0 + r, n = n0 + r;
      xs[c][r] = t < T ? __half2float(X[static_cast<size_t>(t) * K + k0 + c]) : 0.0f;
      ws[c][r] = n < N ? __half2float(W[static_cast<size_t>(n) * K + k0 + c]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRefChunk; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) Y[static_cast<size_t>(t) * N + n] = acc[i][j];
    }
  }
}

// ---- x' = fp16(X / s) ------------------------------------------------------------
// The correctly rounded fp32 quotient rounded to fp16 is the fp16 rounding of
// the exact quotient (a 24-bit intermediate is at least 2 p + 2 for the 11-bit
// fp16 significand).
__global__ void __launch_bounds__(256) divide_activation_kernel(const __half* __restrict__ X,
                                                                const __half* __restrict__ s, long long total, int K,
                                                                __half* __restrict__ Xd) {
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<long long>(gridDim.x) * 256) {
    const int k = static_cast<int>(i % K);
    Xd[i] = __float2half_rn(__fdiv_rn(__half2float(X[i]), __half2float(s[k])));
  }
}

// ---- squared error, per-block fp64 partials ---------------------------------------
// Block b adds (Yq - Y)^2 over elements b * 256 + tid + j * stride in j order,
// then over its threads in a fixed tree; sum_partials_kernel adds the blocks in
// order, so the loss is the same on every run.
__global__ void __launch_bounds__(256) squared_error_kernel(const __half* __restrict__ Yq, const float* __restrict__ Y,
                                                            long long total, double* __restrict__ partial) {
  __shared__ double red[256];
  double acc = 0.0;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<long long>(gridDim.x) * 256) {
    const double d = static_cast<double>(__half2float(Yq[i])) - static_cast<double>(Y[i]);
    acc = fma(d, d, acc);
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int h = 128; h >= 1; h >>= 1) {
    if (threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

// sums[a] = partial[a][0] + partial[a][1] + ... in block order.
__global__ void sum_partials_kernel(const double* __restrict__ partial, int n_alpha, int blocks,
                                    double* __restrict__ sums) {
  const int a = blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= n_alpha) return;
  double acc = 0.0;
  for (int b = 0; b < blocks; ++b) acc += partial[static_cast<size_t>(a) * blocks + b];
  sums[a] = acc;
}

}  // namespace

int search_error_blocks() { return 2 * device_sm_count(); }

cudaError_t launch_reference_gemm(const __half* X, const __half* W, int T, int N, int K, float* Y, cudaStream_t st) {
  const dim3 grid((N + kRefTile - 1) / kRefTile, (T + kRefTile - 1) / kRefTile);
  ref_gemm_kernel<<<grid, 256, 0, st>>>(X, W, T, N, K, Y);
  return cudaGetLastError();
}

cudaError_t launch_divide_activation(const __half* X, const __half* s, int T, int K, __half* Xd, cudaStream_t st) {
  const long long total = static_cast<long long>(T) * K;
  const long long blocks = (total + 255) / 256;
  const int grid = static_cast<int>(blocks < 4 * device_sm_count() ? blocks : 4 * device_sm_count());
  divide_activation_kernel<<<grid, 256, 0, st>>>(X, s, total, K, Xd);
  return cudaGetLastError();
}

cudaError_t launch_squared_error(const __half* Yq, const float* Y, long long total, double* partial, cudaStream_t st) {
  squared_error_kernel<<<search_error_blocks(), 256, 0, st>>>(Yq, Y, total, partial);
  return cudaGetLastError();
}

cudaError_t launch_sum_partials(const double* partial, int n_alpha, double* sums, cudaStream_t st) {
  sum_partials_kernel<<<(n_alpha + 127) / 128, 128, 0, st>>>(partial, n_alpha, search_error_blocks(), sums);
  return cudaGetLastError();
}

}  // namespace w4a16
