// AWQ calibration scale and the quantize + pack kernel.
//
// Pages (by title and section):
//  - "MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide, §AWQ:
//    scale salient input channels by s = s_X^alpha (slides 25-28) and quantize
//    with Q(w) = Delta * Round(w / Delta) per group of 128 (slide 26).
//  - "CMU 11-868 Model Quantization" reading guide, §absmax and zero-point
//    (lecture slide 10): step from (max - min) / (2^N - 1), a rounded zero point,
//    clipping to the code range; a zero range is replaced by 1.
//  - "MIT 6.5940 Lab 4 + Lab 5" reading guide, §Lab 4 setup: calibration
//    statistic = mean |X| per input channel.
//  - Lecture 13 guide, §TinyChat (slide 36): codes packed offline so that the
//    GEMV unpacks them with an AND and a shift (layout v1, include/w4a16.h).
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

// ---------------------------------------------------------------------------
// s[k] = fp16((mean_t |X[t][k]|)^alpha).  One CTA per 64 channels; warp w sums
// the tokens t = w, w + 8, ...  The fp64 sums of fp16 magnitudes are exact for
// T <= 8192 (every term is a multiple of 2^-24 below 2^16), so the order of the
// additions does not change the result.
// ---------------------------------------------------------------------------
constexpr int kAsWarps = 8;
constexpr int kAsChannels = 64;

__global__ void __launch_bounds__(kAsWarps * 32) act_scale_kernel(const __half* __restrict__ X, int T, int K,
                                                                   double alpha, __half* __restrict__ s) {
  __shared__ double part[kAsWarps][kAsChannels];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = blockIdx.x * kAsChannels + 2 * lane;
  double a0 = 0.0, a1 = 0.0;
  for (int t = warp; t < T; t += kAsWarps) {
    const __half* row = X + static_cast<size_t>(t) * K;
    if (k0 < K) a0 += fabs(static_cast<double>(__half2float(row[k0])));
    if (k0 + 1 < K) a1 += fabs(static_cast<double>(__half2float(row[k0 + 1])));
  }
  part[warp][2 * lane] = a0;
  part[warp][2 * lane + 1] = a1;
  __syncthreads();
  if (threadIdx.x < kAsChannels) {
    const int k = blockIdx.x * kAsChannels + threadIdx.x;
    if (k < K) {
      double sum = 0.0;
#pragma unroll
      for (int w = 0; w < kAsWarps; ++w) sum += part[w][threadIdx.x];
      const double mean = sum / static_cast<double>(T);
      s[k] = __double2half(pow(mean, alpha));
    }
  }
}

// ---------------------------------------------------------------------------
// Quantize + pack.  A group of 128 input channels is handled by four lanes (a
// quad): lane q of the quad owns channels 32q .. 32q+31, i.e. four packed words
// of layout v1, read as four 16-byte vectors and written as one.  Group
// statistics are shuffle reductions over the quad (two levels), and the
// per-group step and zero point, worked out by each lane of the quad, are
// shared by 32 values per lane.  Each warp iteration covers eight groups;
// kQpUnroll iterations are loaded before any is computed so that enough bytes
// are in flight.
// ---------------------------------------------------------------------------
constexpr int kQpThreads = 256;
constexpr int kQpQuads = kQpThreads / 4;  // groups per CTA and iteration
constexpr int kQpUnroll = 2;
constexpr int kQpBlocksPerSm = 3;  // resident CTAs per SM the register budget allows

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Round(w / d) with Round = half to even, on the exact quotient.  The IEEE fp32
// quotient decides every half-integer boundary exactly: for fp16 w and d with
// |w / d| < 2^5 a non-tie quotient lies at least 2^-14 from a half-integer,
// far beyond the fp32 rounding error, and an exact tie is representable.
//
// The quotient itself comes from the correctly rounded reciprocal of d (one per
// group): q = w * rcp_rn(d) is within 2^-18 of w / d for |w / d| < 2^5 (two
// fp32 roundings), so rint(q) is already the right decision unless q lies
// within 2^-16 of a half-integer k + 1/2; only then is w compared with
// (k + 1/2) d, which is exact in fp32 (an 11-bit by 7-bit product).  Equality
// is an exact tie (round half to even); otherwise the side of w decides.
// Quotients of 2^5 and more only reach clamped codes.
__device__ __forceinline__ float round_quotient(float w, float d, float inv_d) {
  const float q = w * inv_d;
  const float k = floorf(q);
  if (fabsf(q - k - 0.5f) >= 0x1p-16f) return rintf(q);
  const float t = (k + 0.5f) * d;
  if (w == t) return rintf(k + 0.5f);
  return w > t ? k + 1.0f : k;  // d > 0
}

// 1.5 * 2^23: a float in [2^23, 2^24) has unit spacing, so adding this to a
// value of magnitude below 2^22 rounds it to the nearest integer (ties to
// even), and subtracting it again gives that integer exactly.
constexpr float kRoundMagic = 12582912.0f;

template <int BITS, int MODE, bool HAS_S>
__global__ void __launch_bounds__(kQpThreads, kQpBlocksPerSm) quantize_pack_kernel(const __half* __restrict__ W,
                                                                   const __half* __restrict__ s, int N, int K,
                                                                   uint32_t* __restrict__ qweight,
                                                                   __half* __restrict__ scales,
                                                                   __half* __restrict__ zeros) {
  constexpr int kQmax = (1 << BITS) - 1;
  constexpr int kHalfRange = 1 << (BITS - 1);
  const int Kg = K / kGroup;
  const int Kw = K / 8;
  const long long total = static_cast<long long>(N) * Kg;
  const int ql = threadIdx.x & 3, qd = threadIdx.x >> 2;  // lane in the quad, quad in the CTA
  const int qw = qd & 7;                                   // quad in the warp
  const long long stride = static_cast<long long>(gridDim.x) * kQpQuads;
  long long g0 = static_cast<long long>(blockIdx.x) * kQpQuads + qd;
  // (row, group) of g0 and of the stride, kept in step with g0 without dividing again
  int n0 = static_cast<int>(g0 / Kg), gi0 = static_cast<int>(g0 - static_cast<long long>(n0) * Kg);
  const int sn = static_cast<int>(stride / Kg), sr = static_cast<int>(stride - static_cast<long long>(sn) * Kg);
  auto step = [&](int& n, int& gi) {
    n += sn;
    gi += sr;
    if (gi >= Kg) gi -= Kg, ++n;
  };

  // every quad of a warp runs every iteration (the reductions shuffle over 32 lanes)
  for (; g0 - qw < total; g0 += stride * kQpUnroll) {
    int nn[kQpUnroll], gg[kQpUnroll];
    uint4 wv[kQpUnroll][4];
#pragma unroll
    for (int u = 0; u < kQpUnroll; ++u) {
      nn[u] = u ? nn[u - 1] : n0;
      gg[u] = u ? gg[u - 1] : gi0;
      if (u) step(nn[u], gg[u]);
      const long long g = g0 + u * stride;
#pragma unroll
      for (int c = 0; c < 4; ++c) wv[u][c] = make_uint4(0, 0, 0, 0);
      if (g < total) {
        const __half* wr = W + static_cast<size_t>(nn[u]) * K + gg[u] * kGroup + ql * 32;
#pragma unroll
        for (int c = 0; c < 4; ++c) wv[u][c] = ldg_stream(wr + 8 * c);
      }
    }
    n0 = nn[kQpUnroll - 1];
    gi0 = gg[kQpUnroll - 1];
    step(n0, gi0);
#pragma unroll
    for (int u = 0; u < kQpUnroll; ++u) {
      const long long g = g0 + u * stride;
      // a1: w' = fp16(W * s), the exact product rounded once (mul.rn.f16x2);
      // w2[4c + t] holds channels 32q + 8c + 2t and + 1
      // (s is one row of K values shared by every row of W: read where it is used, from L1)
      __half2 w2[16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        w2[4 * c + 0] = as_h2(wv[u][c].x);
        w2[4 * c + 1] = as_h2(wv[u][c].y);
        w2[4 * c + 2] = as_h2(wv[u][c].z);
        w2[4 * c + 3] = as_h2(wv[u][c].w);
        if (HAS_S && g < total) {
          const uint4 sv = __ldg(reinterpret_cast<const uint4*>(s + gg[u] * kGroup + ql * 32 + 8 * c));
          w2[4 * c + 0] = __hmul2(w2[4 * c + 0], as_h2(sv.x));
          w2[4 * c + 1] = __hmul2(w2[4 * c + 1], as_h2(sv.y));
          w2[4 * c + 2] = __hmul2(w2[4 * c + 2], as_h2(sv.z));
          w2[4 * c + 3] = __hmul2(w2[4 * c + 3], as_h2(sv.w));
        }
      }
      // a2: group statistics over the quad (all 32 lanes take part)
      __half d;
      float zf;
      if (MODE == 0) {
        // (max, -min) in one fp16 pair, so one max per level reduces both
        __half2 hi = w2[0], nlo = __hneg2(w2[0]);
#pragma unroll
        for (int p = 1; p < 16; ++p) {
          hi = __hmax2(hi, w2[p]);
          nlo = __hmax2(nlo, __hneg2(w2[p]));
        }
        __half2 mm = __hmax2(__lows2half2(hi, nlo), __highs2half2(hi, nlo));
#pragma unroll
        for (int o = 2; o >= 1; o >>= 1) mm = __hmax2(mm, as_h2(__shfl_xor_sync(0xffffffffu, as_u32(mm), o)));
        // a3: Delta = fp16((max - min) / (2^N - 1)), the exact quotient rounded
        // once to fp16; a zero step becomes the unit range.  When max - min is
        // exact in fp32 (its TwoSum error term is zero), the correctly rounded
        // fp32 quotient rounded to fp16 is that value: a 24-bit intermediate is
        // at least 2 p + 2 for the 11-bit fp16 significand, so the double
        // rounding is innocuous.  Otherwise (exponents of max and min far
        // apart) the difference and quotient are taken in fp64.
        const float mx = __low2float(mm), nmn = __high2float(mm);  // nmn = -min
        const float diff = mx + nmn;
        const float bv = diff - mx;
        const float err = (mx - (diff - bv)) + (nmn - bv);
        if (err == 0.0f) {
          d = __float2half_rn(__fdiv_rn(diff, static_cast<float>(kQmax)));
        } else {
          d = __double2half((static_cast<double>(mx) + static_cast<double>(nmn)) / static_cast<double>(kQmax));
        }
        if (__heq(d, __float2half(0.0f))) d = __float2half_rn(__fdiv_rn(1.0f, static_cast<float>(kQmax)));
        // z = clamp(Round(-min / Delta), 0, 2^N - 1) as a non-negative integer;
        // the rounding decision is exact (round_quotient), and quotients beyond
        // its range only reach the clamp
        const float dz = __half2float(d);
        zf = fminf(fmaxf(round_quotient(nmn, dz, __frcp_rn(dz)), 0.0f), static_cast<float>(kQmax)) + 0.0f;
      } else {
        __half2 a = __habs2(w2[0]);
#pragma unroll
        for (int p = 1; p < 16; ++p) a = __hmax2(a, __habs2(w2[p]));
        __half am = __hmax(__low2half(a), __high2half(a));
#pragma unroll
        for (int o = 2; o >= 1; o >>= 1) {
          const __half other = __ushort_as_half(
              static_cast<unsigned short>(__shfl_xor_sync(0xffffffffu, static_cast<unsigned>(__half_as_ushort(am)), o)));
          am = __hmax(am, other);
        }
        // a3: Delta = fp16(max|w'| / 2^(N-1)) (a division by a power of two,
        // exact in fp32, then one rounding), z = 2^(N-1)
        d = __float2half_rn(__half2float(am) * (1.0f / static_cast<float>(kHalfRange)));
        if (__heq(d, __float2half(0.0f))) d = __float2half_rn(1.0f / static_cast<float>(kHalfRange));
        zf = static_cast<float>(kHalfRange);
      }
      if (g >= total) continue;
      // a4: u = clamp(Round(w' / Delta) + z, 0, 2^N - 1);  a5: pack into layout v1.
      // Two values at a time (elements 2t, 2t + 1 of a word, bound for bits 4t
      // and 16 + 4t).  q + z = w * inv_d + z is clamped to [-1/4, 2^N - 3/4]
      // (which changes no clamped code) and rounded to an integer by the magic
      // add.  The product is within 2^-19 of w / d for the quotients that are not
      // clamped (|w / d| < 2^5), so the integer is the exact Round unless q + z
      // lies within 2^-16 of a half-integer; then the lane's values are redone
      // with round_quotient, which decides every case exactly.
      const float df = __half2float(d);
      const float inv_d = __frcp_rn(df);
      const uint64_t inv2 = f2_pack(inv_d, inv_d), z2 = f2_pack(zf, zf);
      const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
      // Per word, the two 16-bit halves are summed as integers in floats on a
      // 2^23 base (exact: below 2^16), so their low 16 bits are the packed nibbles.
      uint32_t word[4];
      bool near = false;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint64_t acc = f2_pack(8388608.0f, 8388608.0f);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 wf = __half22float2(w2[4 * c + t]);
          const float2 qz = f2_unpack(f2_fma(f2_pack(wf.x, wf.y), inv2, z2));
          const uint64_t c2 = f2_pack(fminf(fmaxf(qz.x, -0.25f), static_cast<float>(kQmax) + 0.25f),
                                      fminf(fmaxf(qz.y, -0.25f), static_cast<float>(kQmax) + 0.25f));
          const uint64_t u2 = f2_sub(f2_add(c2, magic2), magic2);
          const float2 off = f2_unpack(f2_sub(c2, u2));
          near |= fabsf(off.x) >= 0.5f - 0x1p-16f || fabsf(off.y) >= 0.5f - 0x1p-16f;
          const float sc = static_cast<float>(1 << (4 * t));
          acc = f2_fma(u2, f2_pack(sc, sc), acc);
        }
        const float2 lh = f2_unpack(acc);
        word[c] = __byte_perm(__float_as_uint(lh.x), __float_as_uint(lh.y), 0x5410);
      }
      if (near) {  // a value near a half-integer: the lane's codes again, each decided exactly
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint64_t acc = f2_pack(8388608.0f, 8388608.0f);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 wf = __half22float2(w2[4 * c + t]);
            const uint64_t u2 =
                f2_pack(fminf(fmaxf(round_quotient(wf.x, df, inv_d) + zf, 0.0f), static_cast<float>(kQmax)),
                        fminf(fmaxf(round_quotient(wf.y, df, inv_d) + zf, 0.0f), static_cast<float>(kQmax)));
            const float sc = static_cast<float>(1 << (4 * t));
            acc = f2_fma(u2, f2_pack(sc, sc), acc);
          }
          const float2 lh = f2_unpack(acc);
          word[c] = __byte_perm(__float_as_uint(lh.x), __float_as_uint(lh.y), 0x5410);
        }
      }
      *reinterpret_cast<uint4*>(qweight + static_cast<size_t>(nn[u]) * Kw + gg[u] * 16 + ql * 4) =
          make_uint4(word[0], word[1], word[2], word[3]);
      if (ql == 0) {
        scales[static_cast<size_t>(nn[u]) * Kg + gg[u]] = d;
        zeros[static_cast<size_t>(nn[u]) * Kg + gg[u]] = __float2half_rn(zf);
      }
    }
  }
}

template <int BITS, int MODE, bool HAS_S>
cudaError_t launch_qp(const __half* W, const __half* s, int N, int K, uint32_t* qw, __half* sc, __half* zr,
                      cudaStream_t st) {
  const long long groups = static_cast<long long>(N) * (K / kGroup);
  const long long quads_needed = (groups + kQpUnroll - 1) / kQpUnroll;
  long long blocks = (quads_needed + kQpQuads - 1) / kQpQuads;
  const long long cap = static_cast<long long>(device_sm_count()) * kQpBlocksPerSm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_pack_kernel<BITS, MODE, HAS_S>
      <<<static_cast<unsigned>(blocks), kQpThreads, 0, st>>>(W, s, N, K, qw, sc, zr);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_act_scale(const __half* X, int T, int K, double alpha, __half* s, cudaStream_t st) {
  const int blocks = (K + kAsChannels - 1) / kAsChannels;
  act_scale_kernel<<<blocks, kAsWarps * 32, 0, st>>>(X, T, K, alpha, s);
  return cudaGetLastError();
}

cudaError_t launch_quantize_pack(const __half* W, const __half* s, int N, int K, int bits, int mode,
                                 uint32_t* qw, __half* sc, __half* zr, cudaStream_t st) {
  const bool hs = s != nullptr;
#define W4A16_QP_CASE(B, MO)                                                         \
  if (bits == B && mode == MO)                                                       \
    return hs ? launch_qp<B, MO, true>(W, s, N, K, qw, sc, zr, st)                   \
              : launch_qp<B, MO, false>(W, s, N, K, qw, sc, zr, st);
  W4A16_QP_CASE(4, 0)
  W4A16_QP_CASE(4, 1)
  W4A16_QP_CASE(3, 0)
  W4A16_QP_CASE(3, 1)
#undef W4A16_QP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace w4a16
