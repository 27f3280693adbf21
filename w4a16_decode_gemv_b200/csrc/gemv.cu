// Split-K W4A16 GEMV on CUDA cores for small M (up to kMaxGemvM).
//
//   y[m][n] = sum_g Delta[n][g] * sum_{k in g} (u[n][k] - z[n][g]) * x[m][k]
//
// Decode is a GEMV: every weight is read once per token and the time goes into
// reading weights ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading
// guide, §"why W8A8 is not enough", slides 19-20; "CMU 11-868 Model
// Quantization" guide, §"back to the question").  The kernels stream the packed
// weights at HBM speed and keep the dequantization (an AND/OR per code and one
// subtraction per pair: Lecture 13 guide, §TinyChat, slides 36-37) and the fp32
// multiply-adds under the memory time.
//
// Work split.  The weight is cut into units of R rows x 1024 input channels.
// Units are ordered row-block-major and dealt to all warps of a persistent grid
// (one 16-warp CTA per SM) in contiguous, equal ranges.  Each warp streams its
// own units through a private ring of shared-memory stages filled by bulk copies
// (TMA) that complete on an mbarrier, so every SM keeps ~100-190 KiB of weights
// in flight.  Lane l owns 32 consecutive input channels (a quarter group) of
// each unit row: one 16-byte shared-memory read yields its 4 words.  Partial
// sums stay in registers while a warp's units share a row block; when the row
// block changes the warp reduces them with shuffles and either writes y (it
// covered the whole row) or adds them into the fp32 workspace, the last
// contributor of a row block converting to fp16 and zeroing the workspace behind it.
// Every warp takes at least units_k - 1 units (fewer warps run when the units
// are few), so a row block has at most two contributors; their two fp32 adds
// onto zero commute, and y is the same on every call.
//
// This file holds the kernel for M = 2..4 (and for M = 1 when K is too large
// for the dedicated M = 1 kernel of gemv_m1.cu): units of 4 rows, codes
// unpacked into exact fp16 pairs (u - z) and mixed fp16 x fp16 -> fp32
// multiply-adds.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kUnitWords = 128;  // 1024 input channels per unit row
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
  int warps;           // warps that take units (the first `warps` of the grid)
  int x_bytes;         // shared-memory bytes reserved for the activations
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

// This warp's contiguous range [u0, u0 + cnt) of the units.
__device__ __forceinline__ void warp_range(const GemvArgs& a, int warp, int& u0, int& cnt) {
  const int gw = blockIdx.x * kWarps + warp;
  const int nw = a.warps;
  if (gw >= nw) {
    u0 = a.total_units;
    cnt = 0;
    return;
  }
  const int base = a.total_units / nw;
  const int rem = a.total_units - base * nw;
  u0 = gw * base + min(gw, rem);
  cnt = base + (gw < rem ? 1 : 0);
}

// Issues the bulk copies of unit (rb, kc) of R rows into a ring slot.  Lane r < rows copies row r.
template <int R>
__device__ __forceinline__ void issue_unit(const GemvArgs& a, int rb, int kc, uint8_t* slot, uint64_t* bar,
                                           int lane, uint64_t pol) {
  const int n0 = rb * R;
  const int j0 = kc * kUnitWords;
  const int rows = min(R, a.N - n0);
  const int words = min(kUnitWords, a.Kw - j0);  // a multiple of 16
  const uint32_t row_bytes = static_cast<uint32_t>(words) * 4u;
  if (lane == 0) mbar_arrive_expect_tx(bar, row_bytes * static_cast<uint32_t>(rows));
  __syncwarp();
  if (lane < rows)
    bulk_load_g2s(slot + lane * (kUnitWords * 4), a.qw + static_cast<size_t>(n0 + lane) * a.Kw + j0, row_bytes,
                  bar, pol);
}

// Delta (low 16 bits) and z (high 16 bits) of this lane's group for each unit row.
template <int R>
__device__ __forceinline__ void load_dz(const GemvArgs& a, int rb, int kc, int lane, uint32_t (&dz)[R]) {
  const int g = kc * (kUnitWords / 16) + (lane >> 2);
  const int n0 = rb * R;
  const __half* sp = a.scales + static_cast<size_t>(n0) * a.Kg + g;
  const __half* zp = a.zeros + static_cast<size_t>(n0) * a.Kg + g;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    dz[r] = 0;
    if (n0 + r < a.N && g < a.Kg) dz[r] = ld_nc_u16(sp + r * a.Kg) | (ld_nc_u16(zp + r * a.Kg) << 16);
  }
}

// Sums v[R] (one partial per unit row) over the 32 lanes.  Lane bits 0..log2(R)-1
// select the row whose total the lane returns; lanes 0..R-1 hold distinct rows.
template <int R>
__device__ __forceinline__ float butterfly_rows(const float (&v)[R], int lane, int& row) {
  float t[R];
#pragma unroll
  for (int j = 0; j < R; ++j) t[j] = v[j];
  row = 0;
  int level = 0;
#pragma unroll
  for (int h = R / 2; h >= 1; h /= 2, ++level) {
    const bool b = (lane >> level) & 1;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float keep = b ? t[h + j] : t[j];
      const float send = b ? t[j] : t[h + j];
      t[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << level);
    }
    row += b ? h : 0;
  }
  float k = t[0];
#pragma unroll
  for (int o = R; o < 32; o <<= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
  return k;
}

// Reduces acc[R][MT] over the warp and writes (the warp covered the whole row
// block) or accumulates into the workspace (the last contributor converts).
template <int R, int MT>
__device__ __forceinline__ void flush_rows(const GemvArgs& a, int rb, int contrib, const float (&acc)[R][MT],
                                           int lane) {
  float tot[MT];
  int r = 0;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float v[R];
#pragma unroll
    for (int j = 0; j < R; ++j) v[j] = acc[j][m];
    tot[m] = butterfly_rows<R>(v, lane, r);
  }
  const int n = rb * R + r;
  const bool writer = lane < R && n < a.N;
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
  if (lane == 0)
    last = (atomicAdd(a.ws_cnt + rb, static_cast<uint32_t>(contrib)) + contrib == static_cast<uint32_t>(a.units_k));
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

// Records a timed-out wait and lets the copies already in flight land.
template <int STAGES>
__device__ void bail_out(const GemvArgs& a, uint64_t* bars, int i, int cnt, int lane) {
  if (lane == 0) atomicOr(a.ws_status, kDevWaitTimeout);
  for (int j = i + 1; j < cnt && j < i + STAGES; ++j)
    mbar_wait_bounded(&bars[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u);
}

// ===========================================================================
// M = 1..4 (M = 1 only when the dedicated kernel in gemv_m1.cu cannot run)
// ===========================================================================
constexpr int kRm = 4;
constexpr int kUnitMBytes = kRm * kUnitWords * 4;  // 2 KiB

// XS: x is staged in shared memory (when M*K fp16 fits); otherwise each lane
// reads its activations from global memory (L1/L2 resident).
template <int MT, int STAGES, bool XS>
__global__ void __launch_bounds__(kThreads, 1) gemv_multi_kernel(const GemvArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __half* xs = reinterpret_cast<const __half*>(smem);
  uint8_t* ring = smem + a.x_bytes + warp * (STAGES * kUnitMBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.x_bytes + kWarps * STAGES * kUnitMBytes) + warp * STAGES;

  int u0, cnt;
  warp_range(a, warp, u0, cnt);
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();
  {
    int rb = u0 / a.units_k, kc = u0 - (u0 / a.units_k) * a.units_k;
#pragma unroll
    for (int i = 0; i < STAGES; ++i) {
      if (i < cnt) issue_unit<kRm>(a, rb, kc, ring + i * kUnitMBytes, &bars[i], lane, pol);
      if (++kc == a.units_k) kc = 0, ++rb;
    }
  }

  if (XS) {  // x -> shared memory, once per CTA (M*K fp16; K is a multiple of 128)
    const int chunks = a.M * a.K / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.x);
    uint4* dst = reinterpret_cast<uint4*>(smem);
    for (int c = threadIdx.x; c < chunks; c += kThreads) dst[c] = ld_nc_v4(src + c);
  }
  __syncthreads();
  if (cnt == 0) return;

  float acc[kRm][MT];
#pragma unroll
  for (int r = 0; r < kRm; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
  int rb = u0 / a.units_k;
  int kc = u0 - rb * a.units_k;
  int cur_rb = rb;
  int contrib = 0;
  int rb_f = rb, kc_f = kc;
  for (int j = 0; j < STAGES; ++j)
    if (++kc_f == a.units_k) kc_f = 0, ++rb_f;
  uint32_t dz_next[kRm];
  load_dz<kRm>(a, rb, kc, lane, dz_next);

  for (int i = 0; i < cnt; ++i) {
    const int slot = i % STAGES;
    const uint32_t parity = static_cast<uint32_t>(i / STAGES) & 1u;
    uint32_t dz[kRm];
#pragma unroll
    for (int r = 0; r < kRm; ++r) dz[r] = dz_next[r];
    {
      int rb_n = rb, kc_n = kc + 1;
      if (kc_n == a.units_k) kc_n = 0, ++rb_n;
      if (i + 1 < cnt) load_dz<kRm>(a, rb_n, kc_n, lane, dz_next);
    }
    if (rb != cur_rb) {
      flush_rows<kRm, MT>(a, cur_rb, contrib, acc, lane);
#pragma unroll
      for (int r = 0; r < kRm; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
      cur_rb = rb;
      contrib = 0;
    }

    const int words = min(kUnitWords, a.Kw - kc * kUnitWords);
    const bool active = lane * 4 < words;
    uint32_t xr[MT][16];
    if (active) {
      const int k0 = kc * (kUnitWords * 8) + lane * 32;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < a.M) {
          const uint4* p = reinterpret_cast<const uint4*>((XS ? xs : a.x) + static_cast<size_t>(m) * a.K + k0);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = XS ? p[c] : ld_nc_v4(p + c);
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
      bail_out<STAGES>(a, bars, i, cnt, lane);
      return;
    }

    if (active) {
      const uint4* wq = reinterpret_cast<const uint4*>(ring + slot * kUnitMBytes);
#pragma unroll
      for (int r = 0; r < kRm; ++r) {
        const uint4 w4 = wq[r * (kUnitWords / 4) + lane];
        const __half2 z2 = __half2half2(__ushort_as_half(static_cast<unsigned short>(dz[r] >> 16)));
        const uint32_t nz_lo = as_u32(__hneg2(__hadd2(z2, __floats2half2_rn(1024.0f, 1024.0f))));
        const uint32_t nz_hi = as_u32(__hneg2(__hadd2(z2, __floats2half2_rn(64.0f, 64.0f))));
        const __half2 sixteenth = __floats2half2_rn(0.0625f, 0.0625f);
        // the adds are FMAs with 1: fp16 add issues far slower than FMA on sm_100a
        const __half2 one = __floats2half2_rn(1.0f, 1.0f);
        // (u - z) for the 32 channels, as exact fp16 pairs
        uint32_t dq[16];
        const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t w = wv[c];
          const uint32_t w8 = w >> 8;
          dq[4 * c + 0] = as_u32(__hfma2(as_h2(nib_to_f16x2(w, 0x000F000Fu)), one, as_h2(nz_lo)));
          dq[4 * c + 1] = as_u32(__hfma2(as_h2(nib_to_f16x2(w, 0x00F000F0u)), sixteenth, as_h2(nz_hi)));
          dq[4 * c + 2] = as_u32(__hfma2(as_h2(nib_to_f16x2(w8, 0x000F000Fu)), one, as_h2(nz_lo)));
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
    if (++kc == a.units_k) kc = 0, ++rb;
    // every lane's reads of the stage are ordered before the copy that refills it
    release_stage_reads();
    __syncwarp();
    if (i + STAGES < cnt) issue_unit<kRm>(a, rb_f, kc_f, ring + slot * kUnitMBytes, &bars[slot], lane, pol);
    if (++kc_f == a.units_k) kc_f = 0, ++rb_f;
  }
  flush_rows<kRm, MT>(a, cur_rb, contrib, acc, lane);
}

// ===========================================================================
// host side
// ===========================================================================
int round128(int b) { return (b + 127) / 128 * 128; }

// Largest ring depth (<= 4) whose shared memory fits next to x_bytes.
int pick_stages(int x_bytes, int unit_bytes) {
  for (int st = 4; st >= 2; --st)
    if (x_bytes + kWarps * st * (unit_bytes + 8) <= kMaxSmem) return st;
  return 0;
}

// Launches with programmatic stream serialization when `pdl` is set: the
// kernel may then start while the previous kernel on the stream is finishing,
// and waits for it (griddepcontrol.wait) before touching x, y or the workspace.
template <typename Kern>
cudaError_t launch_kernel(Kern kern, const GemvArgs& a, int grid, int threads, int smem, cudaStream_t st,
                          bool pdl = false) {
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int MT>
cudaError_t launch_multi(const GemvArgs& a, int grid, int stages, cudaStream_t st) {
  const int smem = a.x_bytes + kWarps * stages * (kUnitMBytes + 8);
  if (a.x_bytes == 0) return launch_kernel(gemv_multi_kernel<MT, 4, false>, a, grid, kThreads, smem, st);
  switch (stages) {
    case 4: return launch_kernel(gemv_multi_kernel<MT, 4, true>, a, grid, kThreads, smem, st);
    case 3: return launch_kernel(gemv_multi_kernel<MT, 3, true>, a, grid, kThreads, smem, st);
    case 2: return launch_kernel(gemv_multi_kernel<MT, 2, true>, a, grid, kThreads, smem, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool gemv_supports(int M, int K) {
  (void)K;
  return M >= 1 && M <= kMaxGemvM;
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
  const int sms = device_sm_count();
  const int row_blocks = (p.N + kRm - 1) / kRm;
  a.total_units = row_blocks * a.units_k;
  a.x_bytes = round128(p.M * p.K * 2);
  int stages = pick_stages(a.x_bytes, kUnitMBytes);
  if (stages == 0) {  // x does not fit next to a 2-stage ring: read it from global memory
    a.x_bytes = 0;
    stages = 4;
  }
  // At most two warps contribute to a row block when every warp takes at least
  // units_k - 1 units (a shorter range is what it takes to lie strictly inside
  // a row block), and two partial sums added onto zero give the same fp32 sum in
  // either order: y then does not depend on which contributor comes first.
  a.warps = min(sms * kWarps, a.total_units);
  if (a.units_k > 2) a.warps = max(1, min(a.warps, a.total_units / (a.units_k - 1)));
  const int grid = (a.warps + kWarps - 1) / kWarps;
  switch (p.M) {
    case 1: return launch_multi<1>(a, grid, stages, st);
    case 2: return launch_multi<2>(a, grid, stages, st);
    default: return launch_multi<4>(a, grid, stages, st);
  }
}

}  // namespace w4a16
