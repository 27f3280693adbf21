// Split-K W4A16 GEMV on CUDA cores, for M <= kMaxGemvM.
//
//   y[m][n] = sum_g Delta[n][g] * sum_{k in g} (u[n][k] - z[n][g]) * x[m][k]
//
// Decode is a GEMV: every weight is read once per token and the time goes into
// reading weights ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading
// guide, §"why W8A8 is not enough", slides 19-20; "CMU 11-868 Model
// Quantization" guide, §"back to the question").  So the kernel is built to
// stream the packed weights at HBM speed and to keep the dequantization (AND,
// OR, one fp16 subtract per pair: Lecture 13 guide, §TinyChat, slides 36-37)
// and the fp32 multiply-adds under the memory time.
//
// Work split.  The weight is cut into units of 4 rows x 1024 input channels
// (2 KiB of codes).  Units are ordered row-block-major and dealt to all warps
// of a persistent grid (one 16-warp CTA per SM) in contiguous, equal ranges.
// Each warp streams its own units through a private ring of shared-memory
// stages filled by bulk copies (TMA) that complete on an mbarrier, so every SM
// keeps about 100 KiB of weights in flight.  Lane l owns 32 consecutive input
// channels (a quarter group) of each unit row: one 16-byte shared-memory read
// yields its 4 words.  Partial sums stay in registers while a warp's units
// share a row block; when the row block changes the warp reduces them with
// shuffles and either writes y (it covered the whole row) or adds them into the
// fp32 workspace, the last contributor of a row block converting to fp16 and
// zeroing the workspace behind it.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kUnitRows = 4;
constexpr int kUnitWords = 128;                          // 1024 input channels
constexpr int kUnitBytes = kUnitRows * kUnitWords * 4;   // 2 KiB
constexpr int kMaxSmem = 227 * 1024;

struct GemvArgs {
  const __half* x;
  const uint32_t* qw;
  const __half* scales;
  const __half* zeros;
  __half* y;
  float* ws_acc;       // [M][N]
  uint32_t* ws_cnt;    // [row blocks]
  uint32_t* ws_status;
  int M, N, K;
  int Kw, Kg;          // words and groups per row
  int units_k;         // units per row block
  int total_units;
  int x_bytes;         // shared-memory bytes reserved for x (multiple of 128)
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_nc_u16(const __half* p) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// Issues the bulk copies of unit u into a ring slot.  Lane r < rows copies row r.
__device__ __forceinline__ void issue_unit(const GemvArgs& a, int u, uint8_t* slot, uint64_t* bar, int lane,
                                           uint64_t pol) {
  const int rb = u / a.units_k;
  const int kc = u - rb * a.units_k;
  const int n0 = rb * kUnitRows;
  const int j0 = kc * kUnitWords;
  const int rows = min(kUnitRows, a.N - n0);
  const int words = min(kUnitWords, a.Kw - j0);   // a multiple of 16
  const uint32_t row_bytes = static_cast<uint32_t>(words) * 4u;
  if (lane == 0) mbar_arrive_expect_tx(bar, row_bytes * static_cast<uint32_t>(rows));
  __syncwarp();
  if (lane < rows)
    bulk_load_g2s(slot + lane * (kUnitWords * 4), a.qw + static_cast<size_t>(n0 + lane) * a.Kw + j0, row_bytes,
                  bar, pol);
}

// Delta (low 16 bits) and z (high 16 bits) of this lane's group for each unit row.
__device__ __forceinline__ void load_dz(const GemvArgs& a, int u, int lane, uint32_t (&dz)[kUnitRows]) {
  const int rb = u / a.units_k;
  const int kc = u - rb * a.units_k;
  const int g = kc * (kUnitWords / 16) + (lane >> 2);
#pragma unroll
  for (int r = 0; r < kUnitRows; ++r) {
    const int n = rb * kUnitRows + r;
    dz[r] = 0;
    if (n < a.N && g < a.Kg) {
      const size_t o = static_cast<size_t>(n) * a.Kg + g;
      dz[r] = ld_nc_u16(a.scales + o) | (ld_nc_u16(a.zeros + o) << 16);
    }
  }
}

// Reduces acc[4][MT] over the warp and writes / accumulates the row block.
template <int MT>
__device__ __forceinline__ void flush_rows(const GemvArgs& a, int rb, int contrib, float (&acc)[kUnitRows][MT],
                                           int lane) {
  const bool b0 = lane & 1, b1 = (lane >> 1) & 1;
  float tot[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    // xor 1: even lanes keep rows {0,1}, odd lanes rows {2,3}
    float k0 = b0 ? acc[2][m] : acc[0][m];
    float k1 = b0 ? acc[3][m] : acc[1][m];
    const float s0 = b0 ? acc[0][m] : acc[2][m];
    const float s1 = b0 ? acc[1][m] : acc[3][m];
    k0 += __shfl_xor_sync(0xffffffffu, s0, 1);
    k1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    // xor 2: keep one of the two rows
    float k = b1 ? k1 : k0;
    const float s = b1 ? k0 : k1;
    k += __shfl_xor_sync(0xffffffffu, s, 2);
    k += __shfl_xor_sync(0xffffffffu, k, 4);
    k += __shfl_xor_sync(0xffffffffu, k, 8);
    k += __shfl_xor_sync(0xffffffffu, k, 16);
    tot[m] = k;
  }
  const int r = (b0 ? 2 : 0) + (b1 ? 1 : 0);
  const int n = rb * kUnitRows + r;
  const bool writer = lane < 4 && n < a.N;
  if (contrib == a.units_k) {
    if (writer) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < a.M) a.y[static_cast<size_t>(m) * a.N + n] = __float2half_rn(tot[m]);
    }
    return;
  }
  if (writer) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < a.M) atomicAdd(a.ws_acc + static_cast<size_t>(m) * a.N + n, tot[m]);
  }
  __threadfence();
  __syncwarp();
  uint32_t last = 0;
  if (lane == 0) last = (atomicAdd(a.ws_cnt + rb, static_cast<uint32_t>(contrib)) + contrib ==
                         static_cast<uint32_t>(a.units_k));
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) {
    __threadfence();
    if (writer) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < a.M) {
          const float v = atomicExch(a.ws_acc + static_cast<size_t>(m) * a.N + n, 0.0f);
          a.y[static_cast<size_t>(m) * a.N + n] = __float2half_rn(v);
        }
    }
    if (lane == 0) a.ws_cnt[rb] = 0;
  }
}

template <int MT, int STAGES>
__global__ void __launch_bounds__(kThreads, 1) gemv_w4a16_kernel(const GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __half* xs = reinterpret_cast<const __half*>(smem);
  uint8_t* ring = smem + a.x_bytes + warp * (STAGES * kUnitBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.x_bytes + kWarps * STAGES * kUnitBytes) + warp * STAGES;

  // this warp's contiguous unit range
  const int gw = blockIdx.x * kWarps + warp;
  const int nw = gridDim.x * kWarps;
  const int base = a.total_units / nw;
  const int rem = a.total_units - base * nw;
  const int u0 = gw * base + min(gw, rem);
  const int cnt = base + (gw < rem ? 1 : 0);

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();
#pragma unroll
  for (int i = 0; i < STAGES; ++i)
    if (i < cnt) issue_unit(a, u0 + i, ring + i * kUnitBytes, &bars[i], lane, pol);

  // x -> shared memory, once per CTA (M*K fp16; K is a multiple of 128)
  {
    const int chunks = a.M * a.K / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.x);
    uint4* dst = reinterpret_cast<uint4*>(smem);
    for (int c = threadIdx.x; c < chunks; c += kThreads) dst[c] = ld_nc_v4(src + c);
  }
  __syncthreads();
  if (cnt == 0) return;

  float acc[kUnitRows][MT];
#pragma unroll
  for (int r = 0; r < kUnitRows; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
  int cur_rb = u0 / a.units_k;
  int contrib = 0;
  uint32_t dz_next[kUnitRows];
  load_dz(a, u0, lane, dz_next);

  for (int i = 0; i < cnt; ++i) {
    const int u = u0 + i;
    const int slot = i % STAGES;
    const uint32_t parity = static_cast<uint32_t>(i / STAGES) & 1u;
    const int rb = u / a.units_k;
    const int kc = u - rb * a.units_k;
    uint32_t dz[kUnitRows];
#pragma unroll
    for (int r = 0; r < kUnitRows; ++r) dz[r] = dz_next[r];
    if (i + 1 < cnt) load_dz(a, u + 1, lane, dz_next);

    if (rb != cur_rb) {
      flush_rows<MT>(a, cur_rb, contrib, acc, lane);
#pragma unroll
      for (int r = 0; r < kUnitRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
      cur_rb = rb;
      contrib = 0;
    }

    const int words = min(kUnitWords, a.Kw - kc * kUnitWords);
    const bool active = lane * 4 < words;
    // this lane's 32 activations of each token, as fp16 pairs
    uint32_t xr[MT][16];
    if (active) {
      const int k0 = kc * (kUnitWords * 8) + lane * 32;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < a.M) {
          const uint4* p = reinterpret_cast<const uint4*>(xs + static_cast<size_t>(m) * a.K + k0);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = p[c];
            xr[m][4 * c + 0] = v.x;
            xr[m][4 * c + 1] = v.y;
            xr[m][4 * c + 2] = v.z;
            xr[m][4 * c + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) xr[m][c] = 0;
        }
      }
    }

    if (!mbar_wait_bounded(&bars[slot], parity)) {
      if (lane == 0) atomicOr(a.ws_status, kDevWaitTimeout);
      // let the copies already in flight land before the CTA can exit
      for (int j = i + 1; j < cnt && j < i + STAGES; ++j)
        mbar_wait_bounded(&bars[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u);
      return;
    }

    if (active) {
      const uint4* wq = reinterpret_cast<const uint4*>(ring + slot * kUnitBytes);
#pragma unroll
      for (int r = 0; r < kUnitRows; ++r) {
        const uint4 w4 = wq[r * (kUnitWords / 4) + lane];
        const __half2 z2 = __half2half2(__ushort_as_half(static_cast<unsigned short>(dz[r] >> 16)));
        const uint32_t nz_lo = as_u32(__hneg2(__hadd2(z2, __floats2half2_rn(1024.0f, 1024.0f))));
        const uint32_t nz_hi = as_u32(__hneg2(__hadd2(z2, __floats2half2_rn(64.0f, 64.0f))));
        const __half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
        // (u - z) for the 32 channels, as exact fp16 pairs
        uint32_t dq[16];
        const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t w = wv[c];
          const uint32_t w8 = w >> 8;
          dq[4 * c + 0] = as_u32(__hadd2(as_h2(nib_to_f16x2(w, 0x000F000Fu)), as_h2(nz_lo)));
          dq[4 * c + 1] = as_u32(__hfma2(as_h2(nib_to_f16x2(w, 0x00F000F0u)), sixteenth, as_h2(nz_hi)));
          dq[4 * c + 2] = as_u32(__hadd2(as_h2(nib_to_f16x2(w8, 0x000F000Fu)), as_h2(nz_lo)));
          dq[4 * c + 3] = as_u32(__hfma2(as_h2(nib_to_f16x2(w8, 0x00F000F0u)), sixteenth, as_h2(nz_hi)));
        }
        const float delta = __half2float(__ushort_as_half(static_cast<unsigned short>(dz[r] & 0xFFFFu)));
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < a.M) {
            float p0 = 0.0f, p1 = 0.0f, p2 = 0.0f, p3 = 0.0f;
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              fma2_f16_f32(dq[c], xr[m][c], p0, p1);
              fma2_f16_f32(dq[c + 1], xr[m][c + 1], p2, p3);
            }
            acc[r][m] = fmaf(delta, (p0 + p1) + (p2 + p3), acc[r][m]);
          }
        }
      }
    }
    ++contrib;
    __syncwarp();
    if (i + STAGES < cnt) {
      fence_proxy_async_smem();
      issue_unit(a, u + STAGES, ring + slot * kUnitBytes, &bars[slot], lane, pol);
    }
  }
  flush_rows<MT>(a, cur_rb, contrib, acc, lane);
}

int pick_stages(int x_bytes) {
  for (int st = 4; st >= 2; --st)
    if (x_bytes + kWarps * st * (kUnitBytes + 8) <= kMaxSmem) return st;
  return 0;
}

int x_smem_bytes(int M, int K) { return (M * K * 2 + 127) / 128 * 128; }

template <int MT, int STAGES>
cudaError_t launch_t(const GemvArgs& a, int grid, cudaStream_t st) {
  const int smem = a.x_bytes + kWarps * STAGES * (kUnitBytes + 8);
  auto kern = gemv_w4a16_kernel<MT, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int MT>
cudaError_t launch_m(const GemvArgs& a, int grid, int stages, cudaStream_t st) {
  switch (stages) {
    case 4: return launch_t<MT, 4>(a, grid, st);
    case 3: return launch_t<MT, 3>(a, grid, st);
    case 2: return launch_t<MT, 2>(a, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool gemv_supports(int M, int K) {
  if (M < 1 || M > kMaxGemvM) return false;
  return pick_stages(x_smem_bytes(M, K)) > 0;
}

cudaError_t launch_gemv(const GemmProblem& p, const Workspace& ws, cudaStream_t st) {
  GemvArgs a;
  a.x = p.x;
  a.qw = p.qweight;
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.ws_acc = ws.acc;
  a.ws_cnt = ws.counters;
  a.ws_status = ws.status;
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.Kw = p.K / 8;
  a.Kg = p.K / kGroup;
  a.units_k = (a.Kw + kUnitWords - 1) / kUnitWords;
  const int row_blocks = (p.N + kUnitRows - 1) / kUnitRows;
  a.total_units = row_blocks * a.units_k;
  a.x_bytes = x_smem_bytes(p.M, p.K);
  const int stages = pick_stages(a.x_bytes);
  if (stages == 0) return cudaErrorInvalidValue;
  const int sms = device_sm_count();
  int grid = (a.total_units + kWarps - 1) / kWarps;
  if (grid > sms) grid = sms;
  switch (p.M <= 1 ? 1 : p.M <= 2 ? 2 : 4) {
    case 1: return launch_m<1>(a, grid, stages, st);
    case 2: return launch_m<2>(a, grid, stages, st);
    default: return launch_m<4>(a, grid, stages, st);
  }
}

}  // namespace w4a16
