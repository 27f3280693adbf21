// W4A16 decode GEMV for M = 1 on CUDA cores.
//
//   y[n] = sum_g Delta[n][g] * sum_{k in g} (u[n][k] - z[n][g]) * x[k]
//
// Decode is a GEMV: every weight is read once per token and the time goes into
// reading weights ("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading
// guide, §"why W8A8 is not enough", slides 19-20; "CMU 11-868 Model
// Quantization" guide, §"back to the question").  The codes are unpacked with
// bit masks and the dequantization is fused into the product (Lecture 13 guide,
// §TinyChat, slides 36-37).
//
// Work split.  Row blocks of 4 rows are dealt to the CTAs (one per SM and
// layer) in contiguous, balanced ranges, so a CTA owns whole rows and no
// partial sum leaves the SM.  A CTA's row blocks are cut into units of 4 rows x
// 2048 input channels (4 KiB of codes plus the 4 x 16 Delta and z of those
// rows), and warp w of the CTA takes units w, w + W, w + 2W, ... (W = 8 warps
// when two CTAs share an SM, else 16, or 12 when the staged activations of a
// large K leave room for only 12 rings; see the kernel).  Each warp streams its own
// units through a private ring of shared-memory stages: one lane issues a 2-D
// tensor copy (TMA, box of 4 rows x 256 words, zero fill past the matrix edge)
// per unit and all lanes copy the Delta / z tile with cp.async, all completing
// on the stage's mbarrier.  Many warps issuing copies
// at once keep far more bytes in flight than one producer could.  Each warp
// reduces a unit's 4 row partials across its lanes with shuffles and stores
// them in a shared slot of their own; at the end the CTA adds the slots of each
// row in a fixed order, so y does not depend on timing.
//
// Arithmetic.  Layout v1 puts elements 2t and 2t+1 of a word in nibble slots t
// and t+4, i.e. at bits 4t and 4t+16: the two 16-bit halves of the word carry
// a pair of consecutive elements.  One AND with 0x000F000F isolates elements
// (0, 1) as the fp16 subnormal pair u 2^-24, one with 0x00F000F0 elements (2, 3)
// as u 2^-20 (mantissa bits 4..7); the same two masks on w >> 8 give (4, 5) and
// (6, 7).  Each fp16 pair meets the matching pair of activations, which are the
// input's own fp16 pairs in natural order, in two mixed fp16 x fp16 -> fp32
// FMAs (fma.rn.f32.f16): the products are exact in fp32 and the sums are fp32.
// Per word: 1 shift and 4 ANDs on the ALU pipe (half rate on sm_100) and 8
// mixed FMAs.  The u 2^-20 family is kept in accumulators of its own and scaled
// by 2^-4 once per row.  The zero point is taken out once per row and lane:
// sum (u - z) x = sum u x - z sum x, with 2^-24 sum x of the lane's 64 channels
// staged beside them; 2^24 is folded into Delta.  Lane l owns 64 consecutive
// input channels (8 words, half a group) of each unit row.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kR = 4;                         // rows per unit (= rows per row block)
constexpr int kXBatch = 4;                    // activation words a thread loads at once while staging
constexpr int kMaxSmem = 227 * 1024;
constexpr float kTwo24 = 16777216.0f;        // 2^24

// The geometry of a unit of 4 rows x UW words: UW = 256 (2048 channels, 4 KiB
// of codes) or 128 (1024 channels, 2 KiB).  Lane l owns kWPL = UW / 32
// consecutive words (8 kWPL channels) of each unit row; its staged activations
// are a slice of kSlice 4-byte words: the 8 kWPL fp16 values, 2^-24 times their
// sum, padding (16 bytes, so that 128-bit reads of consecutive slices hit
// distinct banks within a quarter-warp phase).
template <int UW>
struct Geo {
  static constexpr int kUW = UW;
  static constexpr int kWPL = UW / 32;
  static constexpr int kUB = kR * UW * 4;              // codes per unit
  static constexpr int kUG = UW / 16;                  // groups per unit row
  static constexpr int kStage = kUB + 2 * kR * kUG * 2;  // + Delta and z tiles (4 x kUG fp16 each)
  static constexpr int kSliceCh = 8 * kWPL;            // channels per lane slice
  static constexpr int kSlice = 4 * kWPL + 4;          // 4-byte words per slice (4 kWPL + 1 used)
};

struct M1Args {
  const __half* x;
  const uint32_t* qw;
  const __half* scales;
  const __half* zeros;
  __half* y;
  uint32_t* status;  // device status word (wait timeouts)
  int N, K, Kw, Kg;
  int units_k;     // units per row block
  int row_blocks;  // ceil(N / kR)
  int max_units;   // most units any CTA gets
  int x_bytes;     // staged activations (multiple of 128)
  int stages;      // ring depth of each warp
};

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}


// Staged activations: channels are grouped in 64-channel lane slices kSlice
// 4-byte words apart (the 16-byte pad makes the quarter-warp phases of a
// 128-bit read hit distinct banks); a slice holds its 8 words of fp16 x (16
// bytes each) in the owning lane's read order, then 2^-24 times their sum.
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float(static_cast<uint32_t>(127 + e) << 23); }


__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Arrives on `bar` once this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Issues the copies of unit (rb, kc) into a stage: lane 0 the 4 x UW-word
// code box (one TMA op; rows past N and words past K/8 arrive as zeros), lanes
// (tile row, group pair) 4 bytes of the Delta tile and 4 of the z tile with
// cp.async (the group count per row is even, so these pairs are 4-byte
// aligned); every lane arrives once its copies have landed.
template <int UW>
__device__ __forceinline__ void issue_unit(const M1Args& a, const CUtensorMap* tmap, int rb, int kc, uint8_t* dst,
                                           uint64_t* bar, int lane, uint64_t pol) {
  using G = Geo<UW>;
  constexpr int kUB = G::kUB, kUG = G::kUG, kPairs = G::kUG / 2;
  const int n0 = rb * kR;
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(kUB));
    tma_load_2d(dst, tmap, kc * UW, n0, bar, pol);
  }
  const int rows = min(kR, a.N - n0);
  const int words = min(UW, a.Kw - kc * UW);
  const int tr = lane / kPairs, tc = lane % kPairs;  // tile row and group pair of this lane
  if (tr < rows && 2 * tc < words / 16) {
    const size_t o = static_cast<size_t>(n0 + tr) * a.Kg + kc * kUG + 2 * tc;
    __half* tile = reinterpret_cast<__half*>(dst + kUB);
    cp_async_4(tile + tr * kUG + 2 * tc, a.scales + o);
    cp_async_4(tile + kR * kUG + tr * kUG + 2 * tc, a.zeros + o);
  }
  cp_async_arrive(bar);
}

// Two shapes.  CTAS = 2: 8 warps and at most half of an SM's shared memory, so
// that a CTA of the next layer's GEMV can sit on the SM beside one of this
// layer's.  That CTA fills its whole ring before it waits for this layer to
// finish (the weights do not depend on it), so the SM's share of the next
// layer's weights is already streaming while this layer computes, and the
// start-up of a layer (release, activation staging) and the unequal ends of its
// warps no longer leave HBM idle.  CTAS = 1: 16 warps (12 when 16 rings do not
// fit beside the staged activations of a large K) owning the whole SM, with
// only the first stage fetched before the wait.
template <int WARPS, int CTAS, int UW>
__global__ void __launch_bounds__(WARPS * 32, CTAS)
    gemv_m1_kernel(const M1Args a, const __grid_constant__ CUtensorMap tmap) {
  using G = Geo<UW>;
  constexpr int kWarps = WARPS;
  constexpr int kThreads = WARPS * 32;
  constexpr int kUW = UW, kWPL = G::kWPL, kUB = G::kUB, kUG = G::kUG, kStage = G::kStage, kSlice = G::kSlice;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  float* xs = reinterpret_cast<float*>(smem);
  uint8_t* ring = smem + a.x_bytes + static_cast<size_t>(warp) * S * kStage;
  float* part = reinterpret_cast<float*>(smem + a.x_bytes + static_cast<size_t>(kWarps) * S * kStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(part + a.max_units * kR) + warp * S;

  // this CTA's row blocks [rb0, rb1); this warp's units are warp, warp + 8, ...
  const int rb0 = static_cast<int>(static_cast<long long>(blockIdx.x) * a.row_blocks / gridDim.x);
  const int rb1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * a.row_blocks / gridDim.x);
  const int U = (rb1 - rb0) * a.units_k;
  const int dkc = kWarps % a.units_k, drb = kWarps / a.units_k;

  // the next kernel on the stream may start its own prologue right away
  griddep_launch_dependents();
  if (lane == 0) {
    prefetch_tensor_map(&tmap);
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 33);  // expect-tx arrival + 32 cp.async arrivals
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_evict_first_policy();
  // prologue: codes, Delta and z are read-only, so they may be fetched before
  // the previous kernel has finished.  With one CTA per SM only the first
  // stage: the activations are loaded right after griddep_wait and should not
  // queue behind more weights.  With two, the whole ring: the CTA starts while
  // the previous layer still runs, and its copies land long before the wait
  // returns.
  const int pre = CTAS > 1 ? S : 1;
  int rb_f = rb0 + warp / a.units_k, kc_f = warp % a.units_k;
  int jf = warp;
  auto issue_next = [&](int s) {
    issue_unit<UW>(a, &tmap, rb_f, kc_f, ring + static_cast<size_t>(s) * kStage, &full[s], lane, pol);
    jf += kWarps;
    rb_f += drb, kc_f += dkc;
    if (kc_f >= a.units_k) kc_f -= a.units_k, ++rb_f;
  };
  for (int s = 0; s < pre && jf < U; ++s) issue_next(s);

  // x, y and anything earlier kernels produce are touched only after this
  griddep_wait();

  // Word c of x (8 channels) is word c % kWPL of lane slice c / kWPL.  With 8
  // words per lane (UW = 256) the slice's lane (c >> 3) & 31 reads its second
  // 16-byte half first when bit 2 of the lane index is set (see swap1 below),
  // so the words are stored in that order.  Word 4 kWPL of each slice holds
  // 2^-24 times the sum of its channels.  K / 8 is a multiple of 16, so the
  // kWPL words of a slice are kWPL aligned lanes.
  // All of a thread's loads are issued before any is used, so the staging costs
  // one trip to L2 rather than one per word.
  // The loop bound is the warp's first word, so every lane runs every shuffle;
  // lanes past the end contribute nothing.
  for (int c0 = threadIdx.x; c0 - lane < a.K / 8; c0 += kXBatch * kThreads) {
    uint4 v[kXBatch];
#pragma unroll
    for (int q = 0; q < kXBatch; ++q) {
      const int c = c0 + q * kThreads;
      v[q] = c < a.K / 8 ? ld_nc_v4(a.x + 8 * c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < kXBatch; ++q) {
      const int c = c0 + q * kThreads;
      if (c - lane >= a.K / 8) break;  // uniform over the warp
      const bool valid = c < a.K / 8;
      const uint32_t hv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
      // position of word c in its owning lane's read order
      const int jj = kWPL == 8 ? ((c & 7) - 4 * ((c >> 5) & 1)) & 7 : c % kWPL;
      float* slice = xs + (c / kWPL) * kSlice;
      float sum = 0.0f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __half22float2(as_h2(hv[t]));
        sum += f.x + f.y;
      }
      if (valid) *reinterpret_cast<uint4*>(slice + 4 * jj) = v[q];
#pragma unroll
      for (int o = 1; o < kWPL; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (valid && c % kWPL == 0) slice[4 * kWPL] = sum * pow2f(-24);
    }
  }
  __syncthreads();
  // the rest of the ring
  for (int s = pre; s < S && jf < U; ++s) issue_next(s);

  // Lanes with bit 2 set read the second 16-byte half of their 32 bytes of a
  // weight row first, so that the 32-byte lane stride does not put two lanes of
  // a quarter-warp phase on the same banks (their x slices are staged in the
  // same order).
  const int swap1 = kWPL == 8 ? (lane >> 2) & 1 : 0;
  bool failed = false;
  int kc = warp % a.units_k;
  // this lane's staged activations for channel block xkc (reloaded only when the
  // warp's block changes; with 16 warps and K / 2048 dividing 16 it never does)
  int xkc = -1;
  uint32_t xh[4 * kWPL];  // x as fp16 pairs, the lane's kWPL words in read order
  float xsum = 0.0f;      // 2^-24 x the sum of this lane's activations
  for (int j = warp, i = 0; j < U; j += kWarps, ++i) {
    const int s = i % S;
    const uint32_t parity = static_cast<uint32_t>(i / S) & 1u;
    const int ckc = kc;
    kc += dkc;
    if (kc >= a.units_k) kc -= a.units_k;

    const bool act = lane * kWPL < min(kUW, a.Kw - ckc * kUW);
    if (ckc != xkc) {
      xkc = ckc;
      if (act) {
        const float* sl = xs + (ckc * 32 + lane) * kSlice;
        xsum = sl[4 * kWPL];
        const uint4* xb = reinterpret_cast<const uint4*>(sl);
#pragma unroll
        for (int k = 0; k < kWPL; ++k) {
          const uint4 v = xb[k];
          xh[4 * k] = v.x;
          xh[4 * k + 1] = v.y;
          xh[4 * k + 2] = v.z;
          xh[4 * k + 3] = v.w;
        }
      }
    }

    if (!mbar_wait_bounded(&full[s], parity)) {
      if (lane == 0) atomicOr(a.status, kDevWaitTimeout);
      failed = true;
      break;
    }

    float acc[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) acc[r] = 0.0f;
    uint8_t* stage = ring + static_cast<size_t>(s) * kStage;
    if (act) {
      // the lane's kWPL words of each row: one or two 16-byte reads (two: the
      // half nearer the lane's bank first, as its activations were staged)
      const uint4* wq = reinterpret_cast<const uint4*>(stage) + (kWPL / 4) * lane + swap1;
      const __half* tile = reinterpret_cast<const __half*>(stage + kUB) + lane / (16 / kWPL);
#pragma unroll
      for (int r = 0; r < kR; ++r) {
        uint32_t hw[kWPL];
        {
          const uint4 wa = wq[r * (kUW / 4)];
          hw[0] = wa.x, hw[1] = wa.y, hw[2] = wa.z, hw[3] = wa.w;
          if constexpr (kWPL == 8) {
            const uint4 wb = wq[r * (kUW / 4) + 1 - 2 * swap1];
            hw[4] = wb.x, hw[5] = wb.y, hw[6] = wb.z, hw[7] = wb.w;
          }
        }
        const float zf = __half2float(tile[kR * kUG + r * kUG]);
        const float df = __half2float(tile[r * kUG]) * kTwo24;
        // u 2^-24 (bits 0..3 of each 16-bit half) and u 2^-20 (bits 4..7) are
        // fp16 subnormals; their products with x are exact in fp32
        float e0 = 0.0f, e1 = 0.0f, o0 = 0.0f, o1 = 0.0f;
#pragma unroll
        for (int k = 0; k < kWPL; ++k) {
          const uint32_t w = hw[k], w8 = w >> 8;
          fma2_f16_f32(w & 0x000F000Fu, xh[4 * k], e0, e1);
          fma2_f16_f32(w & 0x00F000F0u, xh[4 * k + 1], o0, o1);
          fma2_f16_f32(w8 & 0x000F000Fu, xh[4 * k + 2], e0, e1);
          fma2_f16_f32(w8 & 0x00F000F0u, xh[4 * k + 3], o0, o1);
        }
        // sum (u - z) x = sum u x - z sum x, all scaled by 2^-24
        acc[r] = df * fmaf(-zf, xsum, fmaf(o0 + o1, pow2f(-4), e0 + e1));
      }
    }
    // refill the stage with this warp's unit i + S once every lane's reads are done
    release_stage_reads();
    __syncwarp();
    if (jf < U) issue_next(s);
    // reduce the unit's 4 row partials over the lanes
    const bool b0 = lane & 1, b1 = (lane >> 1) & 1;
    float k0 = b0 ? acc[2] : acc[0];
    float k1 = b0 ? acc[3] : acc[1];
    k0 += __shfl_xor_sync(0xffffffffu, b0 ? acc[0] : acc[2], 1);
    k1 += __shfl_xor_sync(0xffffffffu, b0 ? acc[1] : acc[3], 1);
    float t = b1 ? k1 : k0;
    t += __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 4);
    t += __shfl_xor_sync(0xffffffffu, t, 8);
    t += __shfl_xor_sync(0xffffffffu, t, 16);
    if (lane < 4) part[j * kR + 2 * b0 + b1] = t;  // lane bits -> row 2*b0 + b1
  }
  if (failed) {
    // let this warp's copies in flight land before the CTA can exit
    for (int i2 = 0; i2 < S; ++i2) mbar_wait_bounded(&full[i2], 0u);
  }
  __syncthreads();
  if (failed) return;

  // y[n] = sum over the units of row block (n / 4), in unit order
  const int rows = (rb1 - rb0) * kR;
  for (int i = threadIdx.x; i < rows; i += kThreads) {
    const int n = rb0 * kR + i;
    if (n >= a.N) continue;
    const int rbl = i / kR, r = i - rbl * kR;
    float v = 0.0f;
    for (int c = 0; c < a.units_k; ++c) v += part[(rbl * a.units_k + c) * kR + r];
    a.y[n] = __float2half_rn(v);
  }
}

int round128(int b) { return (b + 127) / 128 * 128; }

int slice_ch(int uw) { return uw == 256 ? Geo<256>::kSliceCh : Geo<128>::kSliceCh; }
int slice_words(int uw) { return uw == 256 ? Geo<256>::kSlice : Geo<128>::kSlice; }
int stage_bytes(int uw) { return uw == 256 ? Geo<256>::kStage : Geo<128>::kStage; }

int x_bytes_for(int K, int uw) { return round128((K / slice_ch(uw)) * slice_words(uw) * 4); }

int smem_for(int warps, int stages, int x_bytes, int max_units, int uw) {
  return x_bytes + warps * stages * stage_bytes(uw) + round128(max_units * kR * 4) + warps * stages * 8;
}

// Shared memory of an SM (228 KiB) less 1 KiB the system reserves per CTA,
// split between two CTAs.
constexpr int kMaxSmemPair = (228 * 1024) / 2 - 1024;

struct M1Config {
  int warps, ctas, uw, stages, smem, grid, max_units;
};

// Two 8-warp CTAs per SM when a CTA's ring holds all of its units, so that the
// whole layer is fetched before the previous layer ends (on B200 that paid at
// 4096 x 4096: 3.65 against 4.23 us per layer; for larger layers the shallower
// rings of two CTAs lost more than the overlap gained: 10.5 against 9.2 us at
// 8192 x 8192).  Else one CTA of 16 warps (12 if 16 two-stage rings do not
// fit); the deepest ring (up to 6 stages) that fits.  Units are 4 rows x 2048
// channels.  (Units of 1024 channels would balance the warps better, 6.5 to 7
// units each instead of 3 or 4, but on B200 they were slower at every layer
// shape, 11.3 against 9.2 us at 8192 x 8192: each unit costs its warp a tensor
// copy issue and a barrier wait, both of which take a fixed, long time.)
// False when nothing fits.
bool m1_config(int N, int K, M1Config& c) {
  const int sms = device_sm_count();
  const int row_blocks = (N + kR - 1) / kR;
  c.grid = min(sms, row_blocks);
  const struct {
    int warps, ctas, uw, limit, max_stages;
  } shapes[3] = {{8, 2, 256, kMaxSmemPair, 6}, {16, 1, 256, kMaxSmem, 6}, {12, 1, 256, kMaxSmem, 6}};
  for (const auto& sh : shapes) {
    const int max_units = ((row_blocks + c.grid - 1) / c.grid) * ((K / 8 + sh.uw - 1) / sh.uw);
    const int xb = x_bytes_for(K, sh.uw);
    if (smem_for(sh.warps, 2, xb, max_units, sh.uw) > sh.limit) continue;
    int st = sh.max_stages;
    while (st > 2 && smem_for(sh.warps, st, xb, max_units, sh.uw) > sh.limit) --st;
    if (sh.ctas == 2 && sh.warps * st < max_units) continue;  // the ring cannot hold the CTA's units
    c.warps = sh.warps;
    c.ctas = sh.ctas;
    c.uw = sh.uw;
    c.stages = st;
    c.max_units = max_units;
    c.smem = smem_for(sh.warps, st, xb, max_units, sh.uw);
    return true;
  }
  return false;
}

}  // namespace

bool gemv_m1_supports(int N, int K) {
  if ((K / kGroup) % 2) return false;  // Delta/z pairs are copied 4 bytes at a time
  M1Config c;
  return m1_config(N, K, c);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda); looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

cudaError_t launch_gemv_m1(const GemmProblem& p, uint32_t* status, cudaStream_t st) {
  M1Args a;
  a.status = status;
  a.x = p.x;
  a.qw = p.qweight;
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.N = p.N;
  a.K = p.K;
  a.Kw = p.K / 8;
  a.Kg = p.K / kGroup;
  M1Config c;
  if (!m1_config(p.N, p.K, c)) return cudaErrorNotSupported;
  a.units_k = (a.Kw + c.uw - 1) / c.uw;
  a.row_blocks = (p.N + kR - 1) / kR;
  const int grid = c.grid;
  a.max_units = c.max_units;
  a.x_bytes = x_bytes_for(p.K, c.uw);
  a.stages = c.stages;
  const int smem = c.smem;

  // qweight as a 2-D tensor of u32: [N rows][K/8 words], boxes of 4 x UW.
  // The map depends only on the pointer and the shape, so the maps of the
  // last few weights this thread launched on are kept (a decode step visits
  // the same layers every token) and encoding is skipped for them.
  struct CachedMap {
    const uint32_t* ptr;
    int n, kw, uw;
    CUtensorMap map;
  };
  constexpr int kMapCache = 64;
  thread_local CachedMap cache[kMapCache] = {};
  thread_local int cache_next = 0;
  const CUtensorMap* tmap = nullptr;
  for (int i = 0; i < kMapCache && !tmap; ++i)
    if (cache[i].ptr == p.qweight && cache[i].n == p.N && cache[i].kw == a.Kw && cache[i].uw == c.uw)
      tmap = &cache[i].map;
  if (!tmap) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.Kw), static_cast<cuuint64_t>(p.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.Kw) * 4};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(c.uw), static_cast<cuuint32_t>(kR)};
    const cuuint32_t estr[2] = {1, 1};
    CachedMap& slot = cache[cache_next];
    if (enc(&slot.map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(p.qweight), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      slot.ptr = nullptr;
      return cudaErrorInvalidValue;
    }
    slot.ptr = p.qweight;
    slot.n = p.N;
    slot.kw = a.Kw;
    slot.uw = c.uw;
    tmap = &slot.map;
    cache_next = (cache_next + 1) % kMapCache;
  }

  auto kern = c.ctas == 2 ? gemv_m1_kernel<8, 2, 256>
                          : (c.warps == 16 ? gemv_m1_kernel<16, 1, 256> : gemv_m1_kernel<12, 1, 256>);
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e == cudaSuccess)
    e = ensure_func_attr(reinterpret_cast<const void*>(kern), cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(c.warps * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a, *tmap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace w4a16
