// W4A8 GEMV for M = 1..4 on CUDA cores, exact in integers.
//
//   acc[m][n] = sum_k x8[m][k] * (u[n][k] * s2[n][g] - zs[n][g])
//             = sum_g ( s2[n][g] * sum_{k in g} u[n][k] x8[m][k]  -  zs[n][g] * sum_{k in g} x8[m][k] )
//   y[m][n]   = fp16( (acc[m][n] * s_x[m]) * s1[n] )     (fp64 products, one rounding each)
//
// The progressive order of "MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment"
// reading guide, §QServe (slides 47-57) multiplies by the group scale before
// subtracting the zero point; on CUDA cores the same integer is reached by
// taking the zero point out once per group: |acc| < K * 127 * 127 < 2^31 for
// K <= 32768, so every partial sum is exact in int32 and the order of addition
// does not matter.
//
// Work split, as the W4A16 decode GEMV: row blocks of 4 rows are dealt to the
// CTAs (one per SM) in contiguous, balanced ranges; a CTA's row blocks are cut
// into units of 4 rows x 2048 inputs (4 KiB of codes plus the 4 x 16 s2 and zs
// bytes), warp w takes units w, w + 16, ...; each warp streams its units' codes
// through a private ring of shared-memory stages (one 2-D tensor copy per unit);
// each lane loads the s2 and zs bytes of its group before it waits for the
// codes.  Lane l owns 64 consecutive inputs (8 words, half a group) of each
// unit row.
//
// Arithmetic.  Layout v1 puts element i of a word in nibble slot [0,4,1,5,2,6,3,7][i];
// so w & 0x0F0F0F0F holds the codes of elements 0, 4, 1, 5 in its four bytes and
// (w >> 4) & 0x0F0F0F0F those of 2, 6, 3, 7.  The activations are staged with
// each block of 8 inputs stored in that order, so one dp4a per half-word
// multiplies four codes by their four activations: per word 1 shift, 2 ANDs and
// 2 dp4a per token.  The sum of the 64 activations of each lane slice is staged
// beside them for the zero point.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kR = 4;                           // rows per unit
constexpr int kUW = 256;                        // words per unit row (2048 inputs)
constexpr int kUB = kR * kUW * 4;               // 4 KiB of codes
constexpr int kUG = kUW / 16;                   // 16 groups per unit row
constexpr int kStage = kUB;                     // codes only
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxSmem = 227 * 1024;

struct W8Args {
  const int8_t* x8;
  const __half* sx;
  const uint32_t* qw;
  const __half* s1;
  const uint8_t* s2;
  const uint8_t* zs;
  __half* y;
  int32_t* acc;      // optional [M][N] exact accumulators (null: not written)
  uint32_t* status;
  int M, N, K, Kw, G;
  int units_k, row_blocks, max_units;
  int x_bytes;       // staged activations and slice sums
  int stages;
};

__device__ __forceinline__ uint32_t ld_nc_u8(const uint8_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// Unit (rb, kc) into a stage: lane 0 issues the 4 x 256-word code box (rows
// past N and words past K/8 arrive as zeros).
__device__ __forceinline__ void issue_unit(const CUtensorMap* tmap, int rb, int kc, uint8_t* dst, uint64_t* bar,
                                           int lane, uint64_t pol) {
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kUB));
    tma_load_2d(dst, tmap, kc * kUW, rb * kR, bar, pol);
  }
}

// Staged activations of token m: the K bytes of x8 with each block of 8 inputs
// in the order 0, 4, 1, 5, 2, 6, 3, 7, then (at xsum) the int32 sum of each
// 64-input slice.
template <int MT>
__global__ void __launch_bounds__(kThreads, 1) w4a8_gemv_kernel(const W8Args a, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  uint8_t* xs = smem;                                   // MT x K bytes
  int32_t* xsum = reinterpret_cast<int32_t*>(smem + MT * a.K);  // MT x K/64
  uint8_t* ring = smem + a.x_bytes + static_cast<size_t>(warp) * S * kStage;
  int32_t* part = reinterpret_cast<int32_t*>(smem + a.x_bytes + static_cast<size_t>(kWarps) * S * kStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(part + a.max_units * kR * MT) + warp * S;

  const int rb0 = static_cast<int>(static_cast<long long>(blockIdx.x) * a.row_blocks / gridDim.x);
  const int rb1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * a.row_blocks / gridDim.x);
  const int U = (rb1 - rb0) * a.units_k;
  const int dkc = kWarps % a.units_k, drb = kWarps / a.units_k;

  griddep_launch_dependents();
  if (lane == 0) {
    prefetch_tensor_map(&tmap);
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();
  int rb_f = rb0 + warp / a.units_k, kc_f = warp % a.units_k;
  int jf = warp;
  auto issue_next = [&](int s) {
    issue_unit(&tmap, rb_f, kc_f, ring + static_cast<size_t>(s) * kStage, &full[s], lane, pol);
    jf += kWarps;
    rb_f += drb, kc_f += dkc;
    if (kc_f >= a.units_k) kc_f -= a.units_k, ++rb_f;
  };
  if (jf < U) issue_next(0);

  griddep_wait();  // x8 may be the previous kernel's output
  // stage x8: thread t takes 8-input blocks t, t + threads, ... of each token;
  // the loop bound is the warp's first block, so every lane runs every shuffle
  for (int m = 0; m < MT; ++m) {
    for (int b0 = threadIdx.x - lane; b0 < a.K / 8; b0 += kThreads) {
      const int b = b0 + lane;
      const bool valid = b < a.K / 8;
      uint2 v = make_uint2(0, 0);
      if (valid && m < a.M) v = *reinterpret_cast<const uint2*>(a.x8 + static_cast<size_t>(m) * a.K + 8 * b);
      // bytes 0..7 = inputs 0..7; stored as 0, 4, 1, 5 | 2, 6, 3, 7
      const uint32_t p0 = __byte_perm(v.x, v.y, 0x5140);
      const uint32_t p1 = __byte_perm(v.x, v.y, 0x7362);
      if (valid) *reinterpret_cast<uint2*>(xs + static_cast<size_t>(m) * a.K + 8 * b) = make_uint2(p0, p1);
      int sm = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        sm += static_cast<int8_t>((v.x >> (8 * j)) & 0xFF) + static_cast<int8_t>((v.y >> (8 * j)) & 0xFF);
      // 8 consecutive lanes hold one 64-input slice (K / 8 is a multiple of 16)
      sm += __shfl_xor_sync(0xffffffffu, sm, 1);
      sm += __shfl_xor_sync(0xffffffffu, sm, 2);
      sm += __shfl_xor_sync(0xffffffffu, sm, 4);
      if (valid && (b & 7) == 0) xsum[m * (a.K / 64) + b / 8] = sm;
    }
  }
  __syncthreads();
  for (int s = 1; s < S && jf < U; ++s) issue_next(s);

  const int swap1 = (lane >> 2) & 1;  // bank spread of the 32-byte lane strides, as the W4A16 GEMV
  bool failed = false;
  int kc = warp % a.units_k;
  // s2 and zs of this lane's group in each row of unit jj (0 past the matrix),
  // fetched two units ahead into one of two register sets (even and odd units of
  // the warp), so that each load has two units' time before its value is read
  auto load_s2zs = [&](int jj, int (&s2o)[kR], int (&zso)[kR]) {
#pragma unroll
    for (int r = 0; r < kR; ++r) s2o[r] = zso[r] = 0;
    if (jj < U) {
      const int kcj = jj % a.units_k;
      const bool actj = lane * 8 < min(kUW, a.Kw - kcj * kUW);
      const int g = kcj * kUG + (lane >> 1);
      const int n0 = (rb0 + jj / a.units_k) * kR;
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const bool in = actj && n0 + r < a.N && g < a.G;
        const size_t o = static_cast<size_t>(n0 + r) * a.G + g;
        s2o[r] = in ? static_cast<int>(ld_nc_u8(a.s2 + o)) : 0;
        zso[r] = in ? static_cast<int>(ld_nc_u8(a.zs + o)) : 0;
      }
    }
  };
  int s2set[2][kR], zsset[2][kR];
  load_s2zs(warp, s2set[0], zsset[0]);
  load_s2zs(warp + kWarps, s2set[1], zsset[1]);
  for (int j2 = warp, i2 = 0; j2 < U && !failed; j2 += 2 * kWarps, i2 += 2)
#pragma unroll
  for (int par = 0; par < 2; ++par) {
    const int j = j2 + par * kWarps, i = i2 + par;
    if (j >= U) break;
    const int s = i % S;
    const uint32_t parity = static_cast<uint32_t>(i / S) & 1u;
    const int ckc = kc;
    kc += dkc;
    if (kc >= a.units_k) kc -= a.units_k;
    const bool act = lane * 8 < min(kUW, a.Kw - ckc * kUW);
    // this lane's 64 activations of each token (16 words, in read order) and their sum
    uint32_t xw[MT][16];
    int xsm[MT];
    if (act) {
      const int slice = ckc * (kUW / 8) + lane;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4* src = reinterpret_cast<const uint4*>(xs + static_cast<size_t>(m) * a.K + 64 * slice);
        const uint4 v0 = src[swap1 * 2], v1 = src[swap1 * 2 + 1], v2 = src[2 - swap1 * 2], v3 = src[3 - swap1 * 2];
        const uint4 vv[4] = {v0, v1, v2, v3};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          xw[m][4 * c] = vv[c].x;
          xw[m][4 * c + 1] = vv[c].y;
          xw[m][4 * c + 2] = vv[c].z;
          xw[m][4 * c + 3] = vv[c].w;
        }
        xsm[m] = xsum[m * (a.K / 64) + slice];
      }
    }
    int s2r[kR], zsr[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      s2r[r] = s2set[par][r];
      zsr[r] = zsset[par][r];
    }
    load_s2zs(j + 2 * kWarps, s2set[par], zsset[par]);
    if (!mbar_wait_bounded(&full[s], parity)) {
      if (lane == 0) atomicOr(a.status, kDevWaitTimeout);
      failed = true;
      break;
    }
    int accr[kR][MT];
    const uint8_t* stage = ring + static_cast<size_t>(s) * kStage;
#pragma unroll
    for (int r = 0; r < kR; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) accr[r][m] = 0;
    if (act) {
      // words 8 lane .. 8 lane + 7 of each row: two 16-byte halves, the half
      // nearer the lane's bank first (its activations were loaded in that order)
      const uint4* wq = reinterpret_cast<const uint4*>(stage) + 2 * lane + swap1;
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const uint4 wa = wq[r * (kUW / 4)];
        const uint4 wb = wq[r * (kUW / 4) + 1 - 2 * swap1];
        const uint32_t hw[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
        const int s2v = s2r[r], zsv = zsr[r];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int d = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            d = __dp4a(static_cast<int>(hw[k] & 0x0F0F0F0Fu), static_cast<int>(xw[m][2 * k]), d);
            d = __dp4a(static_cast<int>((hw[k] >> 4) & 0x0F0F0F0Fu), static_cast<int>(xw[m][2 * k + 1]), d);
          }
          accr[r][m] = s2v * d - zsv * xsm[m];
        }
      }
    }
    release_stage_reads();
    __syncwarp();
    if (jf < U) issue_next(s);
    // sum each (row, token) over the lanes
#pragma unroll
    for (int r = 0; r < kR; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int v = accr[r][m];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) part[(j * kR + r) * MT + m] = v;
      }
  }
  if (failed) {
    for (int i2 = 0; i2 < S; ++i2) mbar_wait_bounded(&full[i2], 0u);
  }
  __syncthreads();
  if (failed) return;

  const int rows = (rb1 - rb0) * kR;
  for (int i = threadIdx.x; i < rows * MT; i += kThreads) {
    const int il = i / MT, m = i - il * MT;
    const int n = rb0 * kR + il;
    if (n >= a.N || m >= a.M) continue;
    const int rbl = il / kR, r = il - rbl * kR;
    int v = 0;
    for (int c = 0; c < a.units_k; ++c) v += part[((rbl * a.units_k + c) * kR + r) * MT + m];
    const double yv = (static_cast<double>(v) * static_cast<double>(__half2float(a.sx[m]))) *
                      static_cast<double>(__half2float(a.s1[n]));
    uint16_t h;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(yv));
    a.y[static_cast<size_t>(m) * a.N + n] = __ushort_as_half(h);
    if (a.acc) a.acc[static_cast<size_t>(m) * a.N + n] = v;
  }
}

int round128(int b) { return (b + 127) / 128 * 128; }

int x_bytes_for(int mt, int K) { return round128(mt * K + mt * (K / 64) * 4); }

int smem_for(int mt, int stages, int x_bytes, int max_units) {
  return x_bytes + kWarps * stages * kStage + round128(max_units * kR * mt * 4) + kWarps * stages * 8;
}

int mt_of(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : 4); }

}  // namespace

bool w4a8_gemv_supports(int M, int N, int K) {
  if (M < 1 || M > 4) return false;
  const int mt = mt_of(M);
  const int row_blocks = (N + kR - 1) / kR;
  const int grid = min(device_sm_count(), row_blocks);
  const int max_units = ((row_blocks + grid - 1) / grid) * ((K / 8 + kUW - 1) / kUW);
  return smem_for(mt, 2, x_bytes_for(mt, K), max_units) <= kMaxSmem;
}

cudaError_t launch_w4a8_gemv(const W4A8Problem& p, uint32_t* status, cudaStream_t st) {
  if (!w4a8_gemv_supports(p.M, p.N, p.K)) return cudaErrorNotSupported;
  W8Args a;
  a.x8 = p.x8;
  a.sx = p.sx;
  a.qw = p.qweight;
  a.s1 = p.s1;
  a.s2 = p.s2;
  a.zs = p.zs;
  a.y = p.y;
  a.acc = p.acc;
  a.status = status;
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.Kw = p.K / 8;
  a.G = p.K / kGroup;
  a.units_k = (a.Kw + kUW - 1) / kUW;
  a.row_blocks = (p.N + kR - 1) / kR;
  const int grid = min(device_sm_count(), a.row_blocks);
  a.max_units = ((a.row_blocks + grid - 1) / grid) * a.units_k;
  const int mt = mt_of(p.M);
  a.x_bytes = x_bytes_for(mt, p.K);
  int stages = 6;
  while (stages > 2 && smem_for(mt, stages, a.x_bytes, a.max_units) > kMaxSmem) --stages;
  a.stages = stages;
  const int smem = smem_for(mt, stages, a.x_bytes, a.max_units);

  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.Kw), static_cast<cuuint64_t>(p.N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.Kw) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kUW), static_cast<cuuint32_t>(kR)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(p.qweight), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  auto kern = mt == 1 ? w4a8_gemv_kernel<1> : (mt == 2 ? w4a8_gemv_kernel<2> : w4a8_gemv_kernel<4>);
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a, tmap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a16
