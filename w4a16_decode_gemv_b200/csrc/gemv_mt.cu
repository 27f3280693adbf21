// W4A16 GEMV for M = 2..4 tokens on CUDA cores.
//
//   y[m][n] = sum_g Delta[n][g] * sum_{k in g} (u[n][k] - z[n][g]) * x[m][k]
//
// A few tokens still leave the product memory-bound: every weight is read once
// for all of them ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading
// guide, §"why W8A8 is not enough", slides 19-20; "CMU 11-868 Model
// Quantization" guide, §"back to the question"), and each code is unpacked once
// and used for every token (dequantization fused into the product: Lecture 13
// guide, §TinyChat, slides 36-37).
//
// Work split.  As for M = 1 (gemv_m1.cu): row blocks of 4 rows are dealt to
// the CTAs (one per SM) in contiguous, balanced ranges; a CTA's row blocks are
// cut into units of 4 rows x 1024 input channels (2 KiB of codes plus the
// 4 x 8 Delta and z), warp w takes units w, w + 8, ..., and streams them
// through a private ring of shared-memory stages filled by one 2-D tensor copy
// (TMA, box of 4 rows x 128 words) plus cp.async copies of the Delta / z tiles.
// Row partial sums stay in the CTA and are added in a fixed order at the end.
//
// Arithmetic (as for M = 1).  A nibble at bit b <= 19 of a word, isolated by
// one AND, reads as the fp32 subnormal u 2^(b-149); the activations of every
// token are staged scaled by 2^(109-b) for each slot, so one packed FMA adds
// u x 2^-40 exactly, and the zero point comes out once per row, lane and token
// as z times 2^-40 sum x.  The unpacking (2 shifts and 16 ANDs per 16 codes) is
// shared by the M tokens; each token adds 8 fma.f32x2.  Lane l owns 32
// consecutive channels (4 words) of each unit row.  For each 2-word block of
// that slice, the lane loads the block's staged activations of all tokens once
// and uses them for the 4 rows of the unit.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kR = 4;                          // rows per unit (= rows per row block)
constexpr int kUW = 128;                       // words per unit row (1024 channels)
constexpr int kUB = kR * kUW * 4;              // 2 KiB of codes per unit
constexpr int kUG = kUW / 16;                  // 8 groups per unit row
constexpr int kStage = kUB + 2 * kR * kUG * 2;  // + Delta and z tiles (4 x 8 fp16 each)
constexpr int kSlice = 36;                     // floats per 32-channel lane slice (+4: sum, pad)
constexpr int kMaxStages = 8;
constexpr int kMaxSmem = 227 * 1024;
constexpr float kTwo40 = 1099511627776.0f;    // 2^40

struct MtArgs {
  const __half* x;
  const uint32_t* qw;
  const __half* scales;
  const __half* zeros;
  __half* y;
  uint32_t* status;  // device status word (wait timeouts)
  int M, N, K, Kw, Kg;
  int units_k;       // units per row block
  int row_blocks;    // ceil(N / kR)
  int max_units;     // most units any CTA gets
  int x_bytes;       // staged activations of one token (multiple of 128)
  int stages;        // ring depth of each warp
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Slot p of layout v1 holds element i = (p < 4 ? 2p : 2(p-4)+1) of its word.
// Bit offset of slot p after the optional shift by 12: 4p (p <= 4), 4p - 12.
__device__ __forceinline__ int slot_bit(int p) { return p <= 4 ? 4 * p : 4 * p - 12; }

__device__ __forceinline__ float pow2f(int e) { return __uint_as_float(static_cast<uint32_t>(127 + e) << 23); }

__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Copies of unit (rb, kc) into a stage: lane 0 the 4 x 128-word code box (one
// TMA op; rows past N and words past K/8 arrive as zeros); lanes 0-15 the
// Delta tile and lanes 16-31 the z tile, a 4-byte pair of groups each.
__device__ __forceinline__ void issue_unit(const MtArgs& a, const CUtensorMap* tmap, int rb, int kc, uint8_t* dst,
                                           uint64_t* bar, int lane, uint64_t pol) {
  const int n0 = rb * kR;
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kUB));
    tma_load_2d(dst, tmap, kc * kUW, n0, bar, pol);
  }
  const int rows = min(kR, a.N - n0);
  const int words = min(kUW, a.Kw - kc * kUW);
  const int arr = lane >> 4, tr = (lane >> 2) & 3, tc = lane & 3;
  if (tr < rows && 2 * tc < words / 16) {
    const size_t o = static_cast<size_t>(n0 + tr) * a.Kg + kc * kUG + 2 * tc;
    __half* tile = reinterpret_cast<__half*>(dst + kUB) + arr * (kR * kUG);
    cp_async_4(tile + tr * kUG + 2 * tc, (arr ? a.zeros : a.scales) + o);
  }
  cp_async_arrive(bar);
}

// Sums v[R] over the 32 lanes (R a power of two, at most 32).  Lane bits
// 0..log2(R)-1 select the value whose total the lane returns (`idx`).
template <int R>
__device__ __forceinline__ float lane_totals(const float (&v)[R], int lane, int& idx) {
  float t[R];
#pragma unroll
  for (int j = 0; j < R; ++j) t[j] = v[j];
  idx = 0;
  int level = 0;
#pragma unroll
  for (int h = R / 2; h >= 1; h /= 2, ++level) {
    const bool hi = (lane >> level) & 1;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float keep = hi ? t[h + j] : t[j];
      const float send = hi ? t[j] : t[h + j];
      t[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << level);
    }
    idx += hi ? h : 0;
  }
  float s = t[0];
#pragma unroll
  for (int o = R; o < 32; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// MT tokens (MT = 2, 3, 4; MP = MT rounded up to a power of two).
template <int MT>
__global__ void __launch_bounds__(kThreads, 1) gemv_mt_kernel(const MtArgs a, const __grid_constant__ CUtensorMap tmap) {
  constexpr int MP = MT <= 2 ? 2 : 4;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  float* xs = reinterpret_cast<float*>(smem);  // MT x x_bytes
  uint8_t* ring = smem + MT * a.x_bytes + static_cast<size_t>(warp) * S * kStage;
  float* part = reinterpret_cast<float*>(smem + MT * a.x_bytes + static_cast<size_t>(kWarps) * S * kStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(part + a.max_units * kR * MP) + warp * S;

  const int rb0 = static_cast<int>(static_cast<long long>(blockIdx.x) * a.row_blocks / gridDim.x);
  const int rb1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * a.row_blocks / gridDim.x);
  const int U = (rb1 - rb0) * a.units_k;
  const int dkc = kWarps % a.units_k, drb = kWarps / a.units_k;

  griddep_launch_dependents();
  if (lane == 0) {
    prefetch_tensor_map(&tmap);
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 33);  // expect-tx arrival + 32 cp.async arrivals
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();
  int rb_f = rb0 + warp / a.units_k, kc_f = warp % a.units_k;
  int jf = warp;
  auto issue_next = [&](int s) {
    issue_unit(a, &tmap, rb_f, kc_f, ring + static_cast<size_t>(s) * kStage, &full[s], lane, pol);
    jf += kWarps;
    rb_f += drb, kc_f += dkc;
    if (kc_f >= a.units_k) kc_f -= a.units_k, ++rb_f;
  };
  // one stage before waiting on the previous kernel (the weights do not depend
  // on it), so that the activation loads below do not queue behind more
  if (jf < U) issue_next(0);

  griddep_wait();

  // x'' of token m = x[m] * 2^(109 - b(slot)), fp32, in pair order: word c of
  // token m is word c & 3 of lane slice c >> 2 (block (c >> 1) & 1, pair half
  // c & 1); float 32 of a slice holds 2^-40 times the sum of its 32 channels.
  // Loads are issued before use; the loop bound is per warp so every lane runs
  // every shuffle (K / 8 is a multiple of 16: the 4 words of a slice are 4
  // aligned lanes of one token).
  const int wpt = a.K / 8;  // words per token
  const int total = MT * wpt;
  for (int c0 = threadIdx.x; c0 - lane < total; c0 += 4 * kThreads) {
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * kThreads;
      const int m = c / wpt;
      v[q] = (c < total && m < a.M) ? ld_nc_v4(a.x + static_cast<size_t>(m) * a.K + 8 * (c - m * wpt))
                                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q * kThreads;
      if (c - lane >= total) break;  // uniform over the warp
      const bool valid = c < total;
      const int m = c / wpt, cw = c - m * wpt;
      const uint32_t hv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
      float* dst = xs + m * (a.x_bytes / 4) + (cw >> 2) * kSlice + 16 * ((cw >> 1) & 1) + (cw & 1);
      float sum = 0.0f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __half22float2(as_h2(hv[t]));
        if (valid) {
          dst[2 * t] = f.x * pow2f(109 - slot_bit(t));
          dst[8 + 2 * t] = f.y * pow2f(109 - slot_bit(4 + t));
        }
        sum += f.x + f.y;
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (valid && (cw & 3) == 0) xs[m * (a.x_bytes / 4) + (cw >> 2) * kSlice + 32] = sum * pow2f(-40);
    }
  }
  __syncthreads();
  for (int s = 1; s < S && jf < U; ++s) issue_next(s);

  bool failed = false;
  int kc = warp % a.units_k;
  for (int j = warp, i = 0; j < U; j += kWarps, ++i) {
    const int s = i % S;
    const uint32_t parity = static_cast<uint32_t>(i / S) & 1u;
    const int ckc = kc;
    kc += dkc;
    if (kc >= a.units_k) kc -= a.units_k;
    const bool act = lane * 4 < min(kUW, a.Kw - ckc * kUW);

    if (!mbar_wait_bounded(&full[s], parity)) {
      if (lane == 0) atomicOr(a.status, kDevWaitTimeout);
      failed = true;
      break;
    }

    float acc[kR * MP];
#pragma unroll
    for (int q = 0; q < kR * MP; ++q) acc[q] = 0.0f;
    uint8_t* stage = ring + static_cast<size_t>(s) * kStage;
    if (act) {
      const uint64_t* wq = reinterpret_cast<const uint64_t*>(stage) + 2 * lane;
      const __half* tile = reinterpret_cast<const __half*>(stage + kUB) + (lane >> 2);
      const float* xl = xs + (ckc * (kUW / 4) + lane) * kSlice;  // this lane's slice of token 0
      uint64_t pa[kR][MT];
#pragma unroll
      for (int r = 0; r < kR; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) pa[r][m] = 0;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint64_t xb[MT][8];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const ulonglong2* src = reinterpret_cast<const ulonglong2*>(xl + m * (a.x_bytes / 4)) + 4 * b;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const ulonglong2 v = src[c];
            xb[m][2 * c] = v.x;
            xb[m][2 * c + 1] = v.y;
          }
        }
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          const uint64_t w = wq[r * (kUW / 2) + b];
          const uint64_t h = f2_pack(static_cast<uint32_t>(w) >> 12, static_cast<uint32_t>(w >> 32) >> 12);
          const uint64_t u[8] = {w & 0x0000000F0000000Full, w & 0x000000F0000000F0ull, w & 0x00000F0000000F00ull,
                                 w & 0x0000F0000000F000ull, w & 0x000F0000000F0000ull, h & 0x00000F0000000F00ull,
                                 h & 0x0000F0000000F000ull, h & 0x000F0000000F0000ull};
#pragma unroll
          for (int p = 0; p < 8; ++p)
#pragma unroll
            for (int m = 0; m < MT; ++m) pa[r][m] = f2_fma(u[p], xb[m][p], pa[r][m]);
        }
      }
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        const float zf = __half2float(tile[kR * kUG + r * kUG]);
        const float df = __half2float(tile[r * kUG]) * kTwo40;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float2 f = f2_unpack(pa[r][m]);
          // sum (u - z) x = sum u x - z sum x, all scaled by 2^-40
          acc[r * MP + m] = df * fmaf(-zf, xl[m * (a.x_bytes / 4) + 32], f.x + f.y);
        }
      }
    }
    release_stage_reads();
    __syncwarp();
    if (jf < U) issue_next(s);
    // totals of the unit's kR x MP partials over the lanes; lane q < kR * MP
    // holds value q = r * MP + m
    int idx;
    const float tot = lane_totals<kR * MP>(acc, lane, idx);
    if (lane < kR * MP) part[j * kR * MP + idx] = tot;
  }
  if (failed) {
    for (int i2 = 0; i2 < S; ++i2) mbar_wait_bounded(&full[i2], 0u);
  }
  __syncthreads();
  if (failed) return;

  // y[m][n] = sum over the units of row block (n / 4), in unit order
  const int rows = (rb1 - rb0) * kR;
  for (int q = threadIdx.x; q < rows * MT; q += kThreads) {
    const int m = q / rows, i = q - m * rows;
    const int n = rb0 * kR + i;
    if (n >= a.N || m >= a.M) continue;
    const int rbl = i / kR, r = i - rbl * kR;
    float v = 0.0f;
    for (int c = 0; c < a.units_k; ++c) v += part[((rbl * a.units_k + c) * kR + r) * MP + m];
    a.y[static_cast<size_t>(m) * a.N + n] = __float2half_rn(v);
  }
}

int round128(int b) { return (b + 127) / 128 * 128; }

int x_bytes_for(int K) { return round128((K / 32) * kSlice * 4); }

int smem_for(int M, int stages, int x_bytes, int max_units) {
  return M * x_bytes + kWarps * stages * kStage + round128(max_units * kR * 4 * 4) + kWarps * stages * 8;
}

int max_units_for(int N, int K, int& grid) {
  const int row_blocks = (N + kR - 1) / kR;
  grid = min(device_sm_count(), row_blocks);
  return ((row_blocks + grid - 1) / grid) * ((K / 8 + kUW - 1) / kUW);
}

template <int MT>
cudaError_t launch_mt(const MtArgs& a, const CUtensorMap& tmap, int grid, int smem, cudaStream_t st) {
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(gemv_mt_kernel<MT>),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
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
  e = cudaLaunchKernelEx(&cfg, gemv_mt_kernel<MT>, a, tmap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool gemv_mt_supports(int M, int N, int K) {
  if (M < 2 || M > 4 || (K / kGroup) % 2) return false;  // Delta/z pairs are copied 4 bytes at a time
  int grid;
  const int mu = max_units_for(N, K, grid);
  return smem_for(M, 2, x_bytes_for(K), mu) <= kMaxSmem;
}

cudaError_t launch_gemv_mt(const GemmProblem& p, uint32_t* status, cudaStream_t st) {
  if (!gemv_mt_supports(p.M, p.N, p.K)) return cudaErrorNotSupported;
  MtArgs a;
  a.x = p.x;
  a.qw = p.qweight;
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.status = status;
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.Kw = p.K / 8;
  a.Kg = p.K / kGroup;
  a.units_k = (a.Kw + kUW - 1) / kUW;
  a.row_blocks = (p.N + kR - 1) / kR;
  int grid;
  a.max_units = max_units_for(p.N, p.K, grid);
  a.x_bytes = x_bytes_for(p.K);
  int stages = kMaxStages;
  while (stages > 2 && smem_for(p.M, stages, a.x_bytes, a.max_units) > kMaxSmem) --stages;
  a.stages = stages;
  const int smem = smem_for(p.M, stages, a.x_bytes, a.max_units);

  // qweight as a 2-D tensor of u32: [N rows][K/8 words], boxes of 4 x 128
  CUtensorMap tmap;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.Kw), static_cast<cuuint64_t>(p.N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.Kw) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kUW), static_cast<cuuint32_t>(kR)};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(p.qweight), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  switch (p.M) {
    case 2: return launch_mt<2>(a, tmap, grid, smem, st);
    case 3: return launch_mt<3>(a, tmap, grid, smem, st);
    default: return launch_mt<4>(a, tmap, grid, smem, st);
  }
}

}  // namespace w4a16
