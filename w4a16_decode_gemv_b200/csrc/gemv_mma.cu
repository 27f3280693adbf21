// W4A16 GEMV for M = 2..8 tokens on the tensor cores, with the dequantized
// weight kept in registers (mma.sync.m16n8k16).
//
//   y[m][n] = sum_g Delta[n][g] * sum_{k in g} (u[n][k] - z[n][g]) * x[m][k]
//
// Small-batch decode reads every weight once per step and the time goes into
// reading weights ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading
// guide, §"why W8A8 is not enough", slides 19-20; "CMU 11-868 Model
// Quantization" guide, §"back to the question").  With a few tokens the
// multiply-adds per weight grow M-fold, which on the CUDA cores makes the
// kernel issue-bound; here they go to the tensor cores.  The 5th-generation
// tcgen05 MMA takes its A operand from tensor or shared memory only, so each
// dequantized weight would be written there and read back once more (per
// weight 4 bytes of on-chip traffic and a barrier hand-off per unit, against
// half a byte from HBM); the register-sourced mma.sync takes the weights
// straight from the registers they are unpacked into, and at 8 tokens its
// throughput (about 600 TFLOP/s measured on B200) is far above what reading
// the weights allows.
//
// Fragments.  An m16n8k16 MMA multiplies 16 weight rows by 16 inputs for 8
// tokens.  Lane l = 4 g + c holds A rows g and g + 8 at two pairs of inputs,
// and B (the activations) for token g at the same two pairs.  Which physical
// inputs an MMA's 16 "k" positions stand for is free, as long as A and B agree:
// lane c takes code word j_c of both of its rows and the activations of the
// same 8 inputs, so one word (8 codes) of each row feeds two MMAs.  Layout v1
// puts the element pairs (0, 1) and (4, 5) of a word at w & 0x000F000F and
// (w >> 8) & 0x000F000F, and (2, 3), (6, 7) at the same masks 0x00F000F0 (16 u):
// OR-ed with 0x6400 they read as the fp16 pairs 1024 + u and 1024 + 16 u, and
// subtracting 1024 + z or 1024 + 16 z leaves the exact integers u - z or
// 16 (u - z) (Lecture 13 guide, §TinyChat, slides 36-37).  The two families go
// to two MMAs with accumulators of their own, and each group's sums are scaled
// once, acc += Delta (s1 + s16 / 16), in fp32: no weight is rounded.
//
// Work split.  Row blocks of 16 rows are dealt to the CTAs in contiguous,
// balanced ranges.  A unit is 16 rows x 256 inputs (two groups, 2 KiB of codes:
// one 128-byte-swizzled tensor copy, so that the lanes' reads of a chunk
// column hit distinct banks), and warp w of the CTA takes units w, w + 16, ...
// of each row block, streaming them through a private ring (the Delta and z of
// the unit's rows come with it by cp.async).  The activations of all tokens are
// staged once per CTA.  Each warp's partial tile of a row block goes to a
// shared slot, and the 16 slots are added in warp order: y does not depend on
// timing.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kRows = 16;                       // rows per row block (the MMA's M)
constexpr int kUW = 32;                         // words per unit row: 256 inputs, two groups
constexpr int kUnitBytes = kRows * kUW * 4;     // 2 KiB of codes
constexpr int kDzBytes = 2 * kRows * 2 * 2;     // Delta and z of the unit: 16 rows x 2 groups each
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMaxStages = 8;
constexpr int kMaxTokens = 8;
constexpr int kSlotFloats = kRows * 8;          // one warp's partial tile: 16 rows x 8 tokens

struct MmaArgs {
  const __half* x;
  const __half* scales;
  const __half* zeros;
  __half* y;
  uint32_t* status;
  int M, N, K, Kg;
  int units_k;     // units per row block
  int row_blocks;  // ceil(N / 16)
  int xrow;        // bytes between staged token rows (2 K + 64: the tokens' 16-byte reads spread over the banks)
  int x_bytes;     // staged activations, rounded up to 128 bytes
  int stages;      // ring depth of each warp
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// c += A B: A 16 x 16 fp16 (row-major fragment), B 16 x 8 fp16 (column-major), c fp32.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (w & mask) | 0x64006400 minus the pair zp: the exact fp16 integers (u - z) or 16 (u - z).
__device__ __forceinline__ uint32_t codes_minus_zero(uint32_t w, uint32_t mask, uint32_t zp) {
  return as_u32(__hsub2(as_h2((w & mask) | 0x64006400u), as_h2(zp)));
}

// Issues unit (rb, kc) into a ring stage: lane 0 the 16 x 32-word code box (one
// tensor copy; rows past N arrive as zeros), lanes 0..15 the unit's two Delta
// values of row rb * 16 + lane and lanes 16..31 the two z values (4-byte
// cp.async: the group count per row is even); every lane arrives once its copy
// has landed.
__device__ __forceinline__ void issue_unit(const MmaArgs& a, const CUtensorMap* tmap, int rb, int kc, uint8_t* codes,
                                           __half* dz, uint64_t* bar, int lane, uint64_t pol) {
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kUnitBytes));
    tma_load_2d(codes, tmap, kc * kUW, rb * kRows, bar, pol);
  }
  const int r = lane & 15;
  const int n = rb * kRows + r;
  if (n < a.N) {
    const size_t o = static_cast<size_t>(n) * a.Kg + 2 * kc;
    cp_async_4(dz + (lane >> 4) * (2 * kRows) + 2 * r, (lane < 16 ? a.scales : a.zeros) + o);
  }
  cp_async_arrive(bar);
}

__global__ void __launch_bounds__(kThreads, 1) gemv_mma_kernel(const MmaArgs a, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ uint8_t smem_raw[];
  // the 128-byte swizzle repeats every 1024 bytes: code stages start on that boundary
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int S = a.stages;
  uint8_t* ring = smem + static_cast<size_t>(warp) * S * kUnitBytes;
  __half* dzr = reinterpret_cast<__half*>(smem + static_cast<size_t>(kWarps) * S * kUnitBytes) +
                static_cast<size_t>(warp) * S * (kDzBytes / 2);
  uint8_t* xs = smem + static_cast<size_t>(kWarps) * S * (kUnitBytes + kDzBytes);
  float* slots = reinterpret_cast<float*>(xs + a.x_bytes);  // [2][kWarps][16 rows][8 tokens]
  uint64_t* full = reinterpret_cast<uint64_t*>(slots + 2 * kWarps * kSlotFloats) + warp * S;

  // this CTA's row blocks [rb0, rb1); this warp's units of each are kc = warp, warp + 16, ...
  const int rb0 = static_cast<int>(static_cast<long long>(blockIdx.x) * a.row_blocks / gridDim.x);
  const int rb1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * a.row_blocks / gridDim.x);
  const int per_rb = warp < a.units_k ? (a.units_k - warp + kWarps - 1) / kWarps : 0;
  const int U = (rb1 - rb0) * per_rb;

  // the next kernel on the stream may start its own prologue right away
  griddep_launch_dependents();
  if (lane == 0) {
    prefetch_tensor_map(&tmap);
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 33);  // expect-tx arrival + 32 cp.async arrivals
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();
  int jf = 0;  // the next of this warp's units to issue
  auto issue_next = [&](int s) {
    const int q = jf / per_rb;
    issue_unit(a, &tmap, rb0 + q, warp + (jf - q * per_rb) * kWarps, ring + s * kUnitBytes, dzr + s * (kDzBytes / 2),
               &full[s], lane, pol);
    ++jf;
  };
  // the weights do not depend on the previous kernel: one stage before the wait
  if (jf < U) issue_next(0);

  // x and y are touched only after this
  griddep_wait();
  // x into shared memory, 16 bytes per thread and step; each thread's loads of a
  // batch are issued before any is stored, so the staging costs one trip to L2
  // per batch rather than one per load
  {
    const int chunks = a.M * (a.K / 8);
    constexpr int kBatch = 8;
    for (int e0 = threadIdx.x; e0 < chunks; e0 += kBatch * kThreads) {
      uint4 v[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int e = e0 + q * kThreads;
        if (e < chunks) v[q] = ld_nc_v4(a.x + static_cast<size_t>(e) * 8);
      }
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        const int e = e0 + q * kThreads;
        if (e < chunks) {
          const int m = e / (a.K / 8), ch = e - m * (a.K / 8);
          *reinterpret_cast<uint4*>(xs + static_cast<size_t>(m) * a.xrow + ch * 16) = v[q];
        }
      }
    }
  }
  __syncthreads();
  for (int s = 1; s < S && jf < U; ++s) issue_next(s);

  // this lane's token (B column).  Past M any staged row will do: B column n
  // reaches only column n of the product, and the columns past M are not stored;
  // every lane loading keeps the loop free of divergent branches.
  const uint8_t* xrow = xs + static_cast<size_t>(g < a.M ? g : 0) * a.xrow;
  bool failed = false;
  int ifail = 0;  // the unit whose wait gave up
  int i = 0;      // units consumed
  for (int rb = rb0; rb < rb1; ++rb) {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // rows g, g + 8 x tokens 2c, 2c + 1
    for (int u = 0; u < per_rb; ++u, ++i) {
      const int kc = warp + u * kWarps;
      const int s = i % S;
      if (!failed && !mbar_wait_bounded(&full[s], static_cast<uint32_t>(i / S) & 1u)) {
        if (lane == 0) atomicOr(a.status, kDevWaitTimeout);
        failed = true;
        ifail = i;
      }
      if (!failed) {
        const uint8_t* st = ring + s * kUnitBytes;
        const __half* dz = dzr + s * (kDzBytes / 2);
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          // the group's step and zero point of rows g and g + 8
          const __half zg = dz[2 * kRows + 2 * g + gi], zg8 = dz[2 * kRows + 2 * (g + 8) + gi];
          const float dg = __half2float(dz[2 * g + gi]), dg8 = __half2float(dz[2 * (g + 8) + gi]);
          const __half k1024 = __ushort_as_half(0x6400u), k16 = __ushort_as_half(0x4C00u);
          const __half z1 = __hadd(zg, k1024), z18 = __hadd(zg8, k1024);
          const __half z16 = __hfma(zg, k16, k1024), z168 = __hfma(zg8, k16, k1024);
          const uint32_t zp1 = as_u32(__halves2half2(z1, z1)), zp18 = as_u32(__halves2half2(z18, z18));
          const uint32_t zp16 = as_u32(__halves2half2(z16, z16)), zp168 = as_u32(__halves2half2(z168, z168));
          float s1[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s16[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            // 16-byte chunk ch of the unit row (words 4 ch .. 4 ch + 3; this lane word c),
            // at chunk ch ^ (row & 7) after the 128-byte swizzle
            const int ch = 4 * gi + jj;
            const uint32_t off = static_cast<uint32_t>(((ch ^ g) << 4) + 4 * c);
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(st + g * 128 + off);
            const uint32_t w8 = *reinterpret_cast<const uint32_t*>(st + (g + 8) * 128 + off);
            // the same 8 inputs of token g: x pairs (0,1) (2,3) (4,5) (6,7)
            const uint4 xv = *reinterpret_cast<const uint4*>(xrow + (kc * kUW + 4 * ch + c) * 16);
            const uint32_t v0 = w0 >> 8, v8 = w8 >> 8;
            mma16816(s1, codes_minus_zero(w0, 0x000F000Fu, zp1), codes_minus_zero(w8, 0x000F000Fu, zp18),
                     codes_minus_zero(v0, 0x000F000Fu, zp1), codes_minus_zero(v8, 0x000F000Fu, zp18), xv.x, xv.z);
            mma16816(s16, codes_minus_zero(w0, 0x00F000F0u, zp16), codes_minus_zero(w8, 0x00F000F0u, zp168),
                     codes_minus_zero(v0, 0x00F000F0u, zp16), codes_minus_zero(v8, 0x00F000F0u, zp168), xv.y, xv.w);
          }
          acc[0] = fmaf(dg, fmaf(s16[0], 0.0625f, s1[0]), acc[0]);
          acc[1] = fmaf(dg, fmaf(s16[1], 0.0625f, s1[1]), acc[1]);
          acc[2] = fmaf(dg8, fmaf(s16[2], 0.0625f, s1[2]), acc[2]);
          acc[3] = fmaf(dg8, fmaf(s16[3], 0.0625f, s1[3]), acc[3]);
        }
      }
      // refill the stage once every lane's reads of it are done
      release_stage_reads();
      __syncwarp();
      if (!failed && jf < U) issue_next(s);
    }
    // this warp's part of row block rb, then the 16 parts added in warp order
    float* sl = slots + ((rb & 1) * kWarps + warp) * kSlotFloats;
    sl[g * 8 + 2 * c] = acc[0];
    sl[g * 8 + 2 * c + 1] = acc[1];
    sl[(g + 8) * 8 + 2 * c] = acc[2];
    sl[(g + 8) * 8 + 2 * c + 1] = acc[3];
    __syncthreads();
    if (threadIdx.x < kRows * kMaxTokens) {
      const int r = threadIdx.x >> 3, m = threadIdx.x & 7;
      const int n = rb * kRows + r;
      if (m < a.M && n < a.N) {
        const float* p = slots + (rb & 1) * kWarps * kSlotFloats + r * 8 + m;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += p[w * kSlotFloats];
        a.y[static_cast<size_t>(m) * a.N + n] = __float2half_rn(v);
      }
    }
  }
  if (failed) {
    // let this warp's copies in flight land before the CTA can exit
    for (int j = ifail; j < jf; ++j) mbar_wait_bounded(&full[j % S], static_cast<uint32_t>(j / S) & 1u);
  }
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

struct MmaConfig {
  int stages, smem, x_bytes, xrow;
};

bool mma_config(int M, int K, MmaConfig& c) {
  if (M < 2 || M > kMaxTokens || K % 256) return false;  // whole units; an even group count per row
  c.xrow = 2 * K + 64;
  c.x_bytes = round_up(M * c.xrow, 128);
  const int fixed = 1024 + c.x_bytes + 2 * kWarps * kSlotFloats * 4;
  for (int st = kMaxStages; st >= 2; --st) {
    const int smem = fixed + kWarps * st * (kUnitBytes + kDzBytes + 8);
    if (smem <= kMaxSmem) {
      c.stages = st;
      c.smem = smem;
      return true;
    }
  }
  return false;
}

}  // namespace

bool gemv_mma_supports(int M, int N, int K) {
  (void)N;
  MmaConfig c;
  return mma_config(M, K, c);
}

cudaError_t launch_gemv_mma(const GemmProblem& p, uint32_t* status, cudaStream_t st) {
  MmaConfig c;
  if (!mma_config(p.M, p.K, c)) return cudaErrorNotSupported;
  MmaArgs a;
  a.x = p.x;
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.status = status;
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.Kg = p.K / kGroup;
  a.units_k = p.K / (8 * kUW);
  a.row_blocks = (p.N + kRows - 1) / kRows;
  a.xrow = c.xrow;
  a.x_bytes = c.x_bytes;
  a.stages = c.stages;
  const int grid = std::min(device_sm_count(), a.row_blocks);

  // qweight as a 2-D tensor of u32 [N rows][K/8 words], boxes of 16 rows x 32
  // words with the 128-byte swizzle; maps of recent weights are kept per thread
  struct CachedMap {
    const uint32_t* ptr;
    int n, kw;
    CUtensorMap map;
  };
  constexpr int kMapCache = 64;
  thread_local CachedMap cache[kMapCache] = {};
  thread_local int cache_next = 0;
  const int Kw = p.K / 8;
  const CUtensorMap* tmap = nullptr;
  for (int i = 0; i < kMapCache && !tmap; ++i)
    if (cache[i].ptr == p.qweight && cache[i].n == p.N && cache[i].kw == Kw) tmap = &cache[i].map;
  if (!tmap) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Kw), static_cast<cuuint64_t>(p.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Kw) * 4};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kUW), static_cast<cuuint32_t>(kRows)};
    const cuuint32_t estr[2] = {1, 1};
    CachedMap& slot = cache[cache_next];
    if (enc(&slot.map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(p.qweight), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      slot.ptr = nullptr;
      return cudaErrorInvalidValue;
    }
    slot.ptr = p.qweight;
    slot.n = p.N;
    slot.kw = Kw;
    tmap = &slot.map;
    cache_next = (cache_next + 1) % kMapCache;
  }

  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(gemv_mma_kernel),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(c.smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, gemv_mma_kernel, a, *tmap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a16
