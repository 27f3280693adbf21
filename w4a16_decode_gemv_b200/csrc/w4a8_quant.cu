// W4A8 with progressive group quantization: the weight and activation
// quantizers ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide,
// §QServe, slides 47-57: 4-bit weights in groups whose scale is applied before
// the zero point, 8-bit per-token activations, int8 tensor cores).
//
// Weights, per output channel n (one warp per row):
//   level 1: s1 = fp16(max_k |W| / 119) (fp16(1/119) for a zero row) and
//            w8 = clip(Round(W / s1), -119, 119);
//   level 2, per group of 128 inputs: mx = max(max w8, 0), mn = min(min w8, 0),
//            s2 = max(1, ceil((mx - mn) / 15)), z2 = clip(Round(-mn / s2), 0, 15),
//            u = clip(Round(w8 / s2) + z2, 0, 15), stored as layout-v1 codes, with
//            s2 and zs = z2 * s2 as bytes.
// Activations, per token m (one CTA per token): s_x = fp16(max_k |x| / 127)
// (fp16(1/127) for a zero token), x8 = clip(Round(x / s_x), -127, 127).
// Round is half-to-even.  Every quotient of two fp16 values is formed in fp64,
// correctly rounded, and then rounded to an integer: for such operands the fp64
// quotient never crosses a half-integer that the exact one does not, so the
// codes are those of exact arithmetic.  The quotients of small integers
// (-mn / s2, w8 / s2) are rounded exactly in integer arithmetic.  fp64 -> fp16
// roundings use cvt.rn.f16.f64 (one rounding, to nearest even).
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kL1 = 119;   // level-1 range
constexpr int kAct = 127;  // activation range

__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return h;
}

__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
  return static_cast<double>(__half2float(__ushort_as_half(h)));
}

// Round(a / b) half-to-even for integers a and b >= 1, exactly.
__device__ __forceinline__ int rint_div(int a, int b) {
  const int m = a < 0 ? -a : a;
  int q = m / b;
  const int r2 = 2 * (m - q * b);
  if (r2 > b || (r2 == b && (q & 1))) ++q;
  return a < 0 ? -q : q;
}

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// Nibble slot of element i of a word in layout v1 (slot p holds i = [0,2,4,6,1,3,5,7][p]).
__device__ __forceinline__ int slot_of(int i) { return (i >> 1) + 4 * (i & 1); }

__global__ void __launch_bounds__(256) w4a8_weight_kernel(const __half* __restrict__ W, int N, int K,
                                                          uint32_t* __restrict__ qweight, __half* __restrict__ s1,
                                                          uint8_t* __restrict__ s2o, uint8_t* __restrict__ zso) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + warp;
  if (n >= N) return;
  const __half* row = W + static_cast<size_t>(n) * K;
  // level 1: the row's largest |w| (exact in fp32)
  float amax = 0.0f;
  for (int k = lane * 8; k < K; k += 256) {
    const uint4 v = *reinterpret_cast<const uint4*>(row + k);
    const uint32_t hv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(as_h2(hv[j]));
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  uint16_t s1h = f64_to_f16_bits(static_cast<double>(amax) / static_cast<double>(kL1));
  if ((s1h & 0x7FFFu) == 0) s1h = f64_to_f16_bits(1.0 / static_cast<double>(kL1));
  const double s1d = f16_bits_to_f64(s1h);
  if (lane == 0) s1[n] = __ushort_as_half(s1h);

  // level 2: lane l takes inputs 4l .. 4l + 3 of each group
  const int G = K / 128;
  for (int g = 0; g < G; ++g) {
    const uint2 v = *reinterpret_cast<const uint2*>(row + g * 128 + 4 * lane);
    const float2 f01 = __half22float2(as_h2(v.x)), f23 = __half22float2(as_h2(v.y));
    const float fv[4] = {f01.x, f01.y, f23.x, f23.y};
    int w8[4];
    int mx = 0, mn = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w8[j] = clampi(static_cast<int>(rint(static_cast<double>(fv[j]) / s1d)), -kL1, kL1);
      mx = max(mx, w8[j]);
      mn = min(mn, w8[j]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const int s2 = max(1, (mx - mn + 14) / 15);
    const int z2 = clampi(rint_div(-mn, s2), 0, 15);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int u = clampi(rint_div(w8[j], s2) + z2, 0, 15);
      word |= static_cast<uint32_t>(u) << (4 * slot_of(4 * (lane & 1) + j));
    }
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    if ((lane & 1) == 0) qweight[static_cast<size_t>(n) * (K / 8) + g * 16 + (lane >> 1)] = word;
    if (lane == 0) {
      s2o[static_cast<size_t>(n) * G + g] = static_cast<uint8_t>(s2);
      zso[static_cast<size_t>(n) * G + g] = static_cast<uint8_t>(z2 * s2);
    }
  }
}

__global__ void __launch_bounds__(256) w4a8_act_kernel(const __half* __restrict__ x, int K, int8_t* __restrict__ x8,
                                                       __half* __restrict__ sx) {
  __shared__ float red[8];
  __shared__ uint16_t s_bits;
  const int m = blockIdx.x;
  const __half* row = x + static_cast<size_t>(m) * K;
  float amax = 0.0f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(__half2float(row[k])));
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x) / 32; ++w) a = fmaxf(a, red[w]);
    uint16_t h = f64_to_f16_bits(static_cast<double>(a) / static_cast<double>(kAct));
    if ((h & 0x7FFFu) == 0) h = f64_to_f16_bits(1.0 / static_cast<double>(kAct));
    s_bits = h;
    sx[m] = __ushort_as_half(h);
  }
  __syncthreads();
  const double sd = f16_bits_to_f64(s_bits);
  int8_t* out = x8 + static_cast<size_t>(m) * K;
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    out[k] = static_cast<int8_t>(
        clampi(static_cast<int>(rint(static_cast<double>(__half2float(row[k])) / sd)), -kAct, kAct));
}

}  // namespace

cudaError_t launch_w4a8_quantize_weight(const __half* W, int N, int K, uint32_t* qweight, __half* s1, uint8_t* s2,
                                        uint8_t* zs, cudaStream_t st) {
  w4a8_weight_kernel<<<(N + 7) / 8, 256, 0, st>>>(W, N, K, qweight, s1, s2, zs);
  return cudaGetLastError();
}

cudaError_t launch_w4a8_quantize_act(const __half* x, int M, int K, int8_t* x8, __half* sx, cudaStream_t st) {
  w4a8_act_kernel<<<M, 256, 0, st>>>(x, K, x8, sx);
  return cudaGetLastError();
}

}  // namespace w4a16
