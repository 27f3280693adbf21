// W4A16 skinny GEMM on the 5th-generation tensor cores (tcgen05) for M = 5..128
// (larger M runs as chunks of 128 tokens, one launch pair per chunk).
//
//   y[m][n] = sum_k x[m][k] * w_hat[n][k],   w_hat = Delta[n][g] * (u[n][k] - z[n][g])
//
// Once several tokens share each weight, the product is a dense contraction and
// belongs on the tensor cores ("MIT 6.5940 Fall 2024 Lecture 13: LLM
// Deployment" reading guide, §SmoothQuant: batching moves the work from
// memory-bound GEMV towards compute).  Up to M = 64 it is still bound by reading
// the packed weights, so the kernel is built to stream them at HBM speed and keep
// the dequantization and the MMAs under that time.
//
// Swap-AB.  The weight rows are the MMA's M dimension (128 rows per MMA) and the
// tokens its N dimension (the token tile MP: M rounded up to 16 up to 64, then
// 96 or 128): D[n][m] = sum_k A[n][k] B[m][k]
// with A = w_hat (fp16) and B = x (fp16, K-major in shared memory), fp32
// accumulators in tensor memory (TMEM lane = weight row, column = token).
//
// w_hat lives in shared memory, in the K-major 128-byte-swizzled layout of an
// MMA operand: the dequantizing thread of a weight row writes its fp16 pairs
// straight into that row's line of a w_hat buffer, and the MMA reads A through
// a shared-memory descriptor, as it reads x.  Tensor memory then holds only the
// accumulators.  (An earlier version wrote w_hat into tensor memory with
// tcgen05.st; on B200 those stores slowed the MMAs' reads of A from tensor
// memory, and this version is faster at every M.)
//
// Work split.  Units are (row block of 256 rows, group of 128 inputs), ordered
// row-block-major and dealt to a persistent grid (one CTA per SM) in contiguous,
// equal ranges.  A CTA accumulates its units of one row block in two 128 x MP
// TMEM accumulators (double-buffered, so the next row block's MMAs overlap the
// read-out of the last).  A CTA that covers a whole row block writes y
// directly; otherwise it writes its fp32 partial tile to one of its two slots
// in the workspace (the row block its range starts in, and the one it ends
// in), and gemm_tc_finalize, launched next on the stream, adds the slots of
// each shared row block in CTA order: y does not depend on timing.
//
// Roles (18 warps):
//   warps 0-15  dequantization and read-out: warp w holds tile t = (w >> 2) & 1
//               (128 rows), TMEM lane quarter q = w & 3 and part p = w >> 3;
//               lane i owns weight row t*128 + q*32 + i of the block, converts
//               words 4p .. 4p + 3 of each 64-input half of a group into w_hat
//               and writes them into one of the shared-memory w_hat buffers;
//               after a row block's MMAs it reads out its rows' accumulator
//               columns;
//   warp 16     one thread issues the tensor copies (TMA) of each unit into a
//               ring of stages: the 256 x 16-word code tile (64-byte swizzle)
//               and the two 64-input halves of the x tile (128-byte swizzle,
//               rows past M zero-filled);
//   warp 17     allocates TMEM; one thread issues tcgen05.mma (8 per 64-input
//               half) and tcgen05.commit.
// Dequantization of a code pair: (w >> 4t) & 0x000F000F | 0x64006400 (one LOP3)
// reads as the fp16 pair 1024 + q; subtracting 1024 + z is exact and the
// multiply by Delta rounds once (Lecture 13 guide, §TinyChat, slides 36-37;
// "CMU 11-868 Model Quantization" guide, §BF16/HFMA2).
//
// Every wait on an mbarrier is bounded; a timeout sets the workspace status word,
// all roles leave their loops, copies and MMAs in flight are waited for, and TMEM
// is freed before the CTA exits.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kDqWarps = 16;                    // dequantization + epilogue warps
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 32 * 18;
constexpr int kRows = 256;                      // weight rows per row block (two MMA tiles)
constexpr int kCodeBytes = kRows * 16 * 4;      // 16 KiB: one group of codes for the block
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMaxStages = 12;
constexpr int kCtrlBytes = 512;

struct TcArgs {
  const uint32_t* qweight;
  const __half* scales;
  const __half* zeros;
  __half* y;
  float4* ws_part;      // [2 x grid slots][MP / 4][256 rows] partial sums
  uint32_t* ws_status;
  int M, N, Kw, Kg;
  int dz_w;             // groups per Delta / z load: the largest of 8, 4, 2, 1 dividing Kg
  int total_units;
  int stages;
};

// ---- tcgen05 / TMEM wrappers ---------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T: A (128 rows x 16 inputs) and B both
// described by shared-memory matrix descriptors.
__device__ __forceinline__ void mma_f16_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

// The w_hat of one code word: 4 fp16 pairs, inputs 8j .. 8j + 7 in order.
struct Word4 {
  uint32_t v[4];
};

// Arrives once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns: thread i gets lane (base + i), columns c..c+7.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (leading offset unused for this layout; encoded as 1).
__device__ __forceinline__ uint64_t sw128_desc(const void* p) {
  const uint32_t a = smem_u32(p);
  const uint32_t lo = ((a >> 4) & 0x3FFFu) | (1u << 16);
  const uint32_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// kind::f16 instruction descriptor: fp32 D, fp16 A and B, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// ---- waits, arrivals, barriers --------------------------------------------------
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait that also gives up as soon as another role has given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                                              uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, kDevWaitTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t lop3_nib(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
  return r;
}

// W consecutive fp16 values (W = 1, 2, 4 or 8, the address aligned to 2W bytes)
// into the low halves of w[0..3], lowest address first.
__device__ __forceinline__ void ld_nc_halves(const __half* p, int W, uint32_t (&w)[4]) {
  w[0] = w[1] = w[2] = w[3] = 0;
  if (W == 8)
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "l"(p));
  else if (W == 4)
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "l"(p));
  else if (W == 2)
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(w[0]) : "l"(p));
  else
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(w[0]) : "l"(p));
}

// The idx-th fp16 value (0..7) of four packed words, zero-extended.
__device__ __forceinline__ uint32_t pick_half(const uint32_t (&w)[4], int idx) {
  const uint32_t v = (idx & 4) ? ((idx & 2) ? w[3] : w[2]) : ((idx & 2) ? w[1] : w[0]);
  return (idx & 1) ? (v >> 16) : (v & 0xFFFFu);
}

__device__ __forceinline__ void sts128(uint32_t addr, const Word4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.v[0]), "r"(v.v[1]), "r"(v.v[2]),
               "r"(v.v[3])
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// (1024 + u) - (1024 + z) = u - z exactly, computed as an FMA with 1 (the fp16
// add and subtract instructions issue far slower than FMA on sm_100a), then one
// rounding in the multiply by Delta.  nz = -(1024 + z).
__device__ __forceinline__ uint32_t dq_pair(uint32_t v, __half2 nz, __half2 dd) {
  return as_u32(__hmul2(__hfma2(as_h2(lop3_nib(v)), __float2half2_rn(1.0f), nz), dd));
}

__device__ __forceinline__ Word4 dq_word(uint32_t w, __half2 zz, __half2 dd) {
  return Word4{{dq_pair(w, zz, dd), dq_pair(w >> 4, zz, dd), dq_pair(w >> 8, zz, dd), dq_pair(w >> 12, zz, dd)}};
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Tensor memory holds only the accumulators: 2 buffers x 2 tiles x MP columns,
// allocated as the next power of two of at least 32 columns.
__host__ __device__ constexpr uint32_t tmem_cols(int mp) {
  return 4 * mp <= 32 ? 32u : 4 * mp <= 64 ? 64u : 4 * mp <= 128 ? 128u : 4 * mp <= 256 ? 256u : 512u;
}
// w_hat lives in shared memory: kABufs buffers, each one 64-input half of a
// unit (2 tiles x 128 rows x 128 bytes, K-major with the 128-byte swizzle, the
// layout the MMA's shared-memory descriptor reads).
constexpr int kABufs = 4;
constexpr int kMaxABufs = kABufs;
constexpr int kTileBytes = 128 * 128;
constexpr int kABufBytes = 2 * kTileBytes;

// Unit u of the range partition: the CTA whose range holds it.
__host__ __device__ __forceinline__ int owner_cta(int u, int base, int rem) {
  const int big = rem * (base + 1);
  return u < big ? u / (base + 1) : rem + (u - big) / base;
}

template <int MP>
__global__ void __maxnreg__(96)
    gemm_tc_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tx) {
  constexpr int kXHalf = MP * 128;                // one 64-input half of the x tile
  constexpr int kStageBytes = kCodeBytes + 2 * kXHalf;
  constexpr uint32_t kIdesc = idesc_f16(MP);
  constexpr uint32_t kTmemCols = tmem_cols(MP);
  static_assert(kABufs >= 4, "a unit writes two w_hat buffers; four keep the MMAs one unit behind");
  static_assert(kStageBytes % 1024 == 0, "w_hat buffers must stay 1024-byte aligned");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages;
  uint8_t* stages = smem;                        // S x kStageBytes: code tile, then x tile
  uint8_t* abuf = stages + S * kStageBytes;      // kABufs x kABufBytes of w_hat
  uint64_t* bars = reinterpret_cast<uint64_t*>(abuf + kABufs * kABufBytes);
  uint64_t* full = bars;                         // [S] codes and x landed
  uint64_t* rempty = bars + kMaxStages;          // [S] codes read and x consumed
  uint64_t* wfull = bars + 2 * kMaxStages;       // [kABufs] w_hat half written to shared memory
  uint64_t* wempty = wfull + kMaxABufs;          // [kABufs] w_hat half consumed by the MMAs
  uint64_t* afull = wempty + kMaxABufs;          // [2] accumulator complete
  uint64_t* aempty = afull + 2;                  // [2] accumulator read out
  uint64_t* tdown = aempty + 2;                  // teardown: all MMAs complete
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tdown + 1);
  volatile uint32_t* abort_flag = tslot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int base = a.total_units / static_cast<int>(gridDim.x);
  const int rem = a.total_units - base * static_cast<int>(gridDim.x);
  const int bx = static_cast<int>(blockIdx.x);
  const int u0 = bx * base + min(bx, rem);
  const int cnt = base + (bx < rem ? 1 : 0);
  const int rb0 = u0 / a.Kg;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&rempty[s], kDqWarps + 1);  // dequantization warps + 1 MMA commit
    }
    for (int b = 0; b < kABufs; ++b) {
      mbar_init(&wfull[b], kDqWarps);
      mbar_init(&wempty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], kDqWarps);
    }
    mbar_init(tdown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tslot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  // the next kernel on the stream (the partial-sum finalize) may begin launching
  griddep_launch_dependents();

  if (warp == kProducerWarp) {
    // ---------------- producer: tensor copies of codes and x ----------------
    if (lane == 0) {
      const uint64_t pol_q = l2_evict_first_policy();
      const uint64_t pol_x = l2_evict_last_policy();
      auto code_copy = [&](int i) {
        const int u = u0 + i, rb = u / a.Kg, g = u - rb * a.Kg;
        const int s = i % S;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(stages + s * kStageBytes, &tq, g * 16, rb * kRows, &full[s], pol_q);
      };
      auto x_copy = [&](int i) {
        const int g = (u0 + i) % a.Kg;
        const int s = i % S;
        uint8_t* xs = stages + s * kStageBytes + kCodeBytes;
        tma_load_2d(xs, &tx, g * 128, 0, &full[s], pol_x);
        tma_load_2d(xs + kXHalf, &tx, g * 128 + 64, 0, &full[s], pol_x);
      };
      // the weights do not depend on the previous kernel: start streaming them first
      const int pre = min(S, cnt);
      for (int i = 0; i < pre; ++i) code_copy(i);
      griddep_wait();  // x may be the previous kernel's output
      for (int i = 0; i < pre; ++i) x_copy(i);
      int issued = pre;
      for (int i = pre; i < cnt; ++i) {
        const int s = i % S;
        if (!wait_or_abort(&rempty[s], static_cast<uint32_t>(i / S - 1) & 1u, abort_flag, a.ws_status)) break;
        code_copy(i);
        x_copy(i);
        issued = i + 1;
      }
      // copies still in flight must land before the CTA may exit
      for (int j = max(0, issued - S); j < issued; ++j)
        mbar_wait_bounded(&full[j % S], static_cast<uint32_t>(j / S) & 1u);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool any = false;
      int hb = 0, f = 0;
      for (int i = 0; i < cnt; ++i) {
        const int s = i % S;
        const int g = (u0 + i) % a.Kg;
        const bool first = (i == 0) || (g == 0);
        const bool last = (i == cnt - 1) || (g == a.Kg - 1);
        const int ab = f & 1;
        if (first && f >= 2 && !wait_or_abort(&aempty[ab], static_cast<uint32_t>(f / 2 - 1) & 1u, abort_flag, a.ws_status))
          break;
        if (!wait_or_abort(&full[s], static_cast<uint32_t>(i / S) & 1u, abort_flag, a.ws_status)) break;
        bool ok = true;
        const uint8_t* xs = stages + s * kStageBytes + kCodeBytes;
        for (int h = 0; h < 2; ++h) {
          const int b = hb % kABufs;
          if (!wait_or_abort(&wfull[b], static_cast<uint32_t>(hb / kABufs) & 1u, abort_flag, a.ws_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Addresses computed once per half: the B descriptor's start-address
          // field advances by 32 bytes (2 in 16-byte units) per 16 inputs, A
          // and D are tensor-memory columns at fixed offsets.  This thread
          // shares its scheduler with dequantizing warps, so few instructions
          // per MMA matter.
          const uint64_t bd0 = sw128_desc(xs + h * kXHalf);
          const uint64_t ad0 = sw128_desc(abuf + b * kABufBytes);
          const uint32_t d0 = tbase + static_cast<uint32_t>(ab * 2 * MP);
          const bool acc0 = !(first && h == 0);
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(d0 + t * MP, ad0 + t * (kTileBytes >> 4) + 2 * kk, bd0 + 2 * kk, kIdesc, kk > 0 || acc0);
          any = true;
          mma_commit(&wempty[b]);
          ++hb;
        }
        if (!ok) break;
        mma_commit(&rempty[s]);
        if (last) {
          mma_commit(&afull[ab]);
          ++f;
        }
      }
      if (any) {
        mma_commit(tdown);
        mbar_wait_bounded(tdown, 0);
      }
    }
  } else if (warp < kDqWarps) {
    // ---------------- dequantization and epilogue ----------------
    // Warp w: tile t = (w >> 2) & 1, TMEM lane quarter q = w & 3, part p = w >> 3.
    // Its lanes own rows t*128 + q*32 + lane of the block; of each 64-input half
    // of a group it converts words 4p .. 4p + 3 (TMEM columns 16p .. 16p + 15 of
    // the tile), and at the end of a row block it reads out accumulator columns
    // p*MP/2 .. (p+1)*MP/2 - 1 of its rows.
    const int t = (warp >> 2) & 1, q = warp & 3, p = warp >> 3;
    const int rloc = t * 128 + q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    // this lane's w_hat row in a buffer: tile t, row q * 32 + lane, 128 bytes
    // with the 16-byte chunk j at j ^ (row & 7)
    const int arow = q * 32 + lane;
    const uint32_t arow0 = smem_u32(abuf) + static_cast<uint32_t>(t * kTileBytes + arow * 128);
    const uint32_t asw = static_cast<uint32_t>(arow & 7);
    const uint32_t st0 = smem_u32(stages);
    const uint32_t sw_ld = static_cast<uint32_t>((rloc >> 1) & 3);
    // Delta and z come a block of W groups at a time (W = 1, 2, 4 or 8 divides
    // K / 128, so the W values of a row are one aligned load), one block ahead.
    const int W = a.dz_w;
    uint32_t dc[4], zc[4], dn[4], zn[4];
    auto issue_dz = [&](int ub) {
      const int rb = ub / a.Kg, g = ub - rb * a.Kg, g0 = g & ~(W - 1);
      const int n = rb * kRows + rloc;
      if (n < a.N) {
        const size_t o = static_cast<size_t>(n) * a.Kg + g0;
        ld_nc_halves(a.scales + o, W, dn);
        ld_nc_halves(a.zeros + o, W, zn);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) dn[j] = zn[j] = 0;
      }
    };
    int hb = 0, f = 0, start = 0;
    int pend = -1, pend_rb = 0, pend_contrib = 0;  // a row block whose accumulator awaits read-out
    bool ok = true;
    // Read-out of the accumulator of flush number f (row block rb, `contrib` units).
    auto flush = [&](int fl, int rb, int contrib) {
      const int ab = fl & 1;
      const bool okw = wait_or_abort(&afull[ab], static_cast<uint32_t>(fl / 2) & 1u, abort_flag, a.ws_status);
      if (__any_sync(0xffffffffu, !okw)) {
        ok = false;
        return;
      }
      tc_fence_after();
      const bool owner = contrib == a.Kg;
      const int n = rb * kRows + rloc;
      // a CTA has at most two partial row blocks: the one its range starts in
      // (slot 0) and the one it ends in (slot 1); blocks in between are whole
      float4* slot = a.ws_part + static_cast<size_t>(bx * 2 + (rb == rb0 ? 0 : 1)) * (kRows * MP / 4);
#pragma unroll
      for (int c = 0; c < MP / 16; ++c) {
        const int m0 = p * (MP / 2) + c * 8;
        float v[8];
        tmem_ld8(tbase + lane_addr + static_cast<uint32_t>(ab * 2 * MP + t * MP + m0), v);
        if (n < a.N) {
          if (owner) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (m0 + j < a.M) a.y[static_cast<size_t>(m0 + j) * a.N + n] = __float2half_rn(v[j]);
          } else {
            slot[(m0 / 4) * kRows + rloc] = make_float4(v[0], v[1], v[2], v[3]);
            slot[(m0 / 4 + 1) * kRows + rloc] = make_float4(v[4], v[5], v[6], v[7]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[ab]);
    };
    const int uend = u0 + cnt;
    int cur_end = u0;  // the Delta / z block in dc / zc covers units up to cur_end - 1
    issue_dz(u0);
    for (int i = 0; i < cnt && ok; ++i) {
      const int u = u0 + i;
      const int g = u % a.Kg;
      if (u >= cur_end) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          dc[j] = dn[j];
          zc[j] = zn[j];
        }
        cur_end = u + min(W - (g & (W - 1)), a.Kg - g);
        if (cur_end < uend) issue_dz(cur_end);
      }
      const int s = i % S;
      const bool okf = wait_or_abort(&full[s], static_cast<uint32_t>(i / S) & 1u, abort_flag, a.ws_status);
      if (__any_sync(0xffffffffu, !okf)) {
        ok = false;
        break;
      }
      const uint32_t row = st0 + static_cast<uint32_t>(s * kStageBytes + rloc * 64);
      const uint4 c0 = lds128(row + ((static_cast<uint32_t>(p) ^ sw_ld) << 4));
      const uint4 c1 = lds128(row + ((static_cast<uint32_t>(2 + p) ^ sw_ld) << 4));
      release_stage_reads();
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[s]);  // codes are in registers
      const uint32_t dv = pick_half(dc, g & (W - 1)), zv = pick_half(zc, g & (W - 1));
      const __half2 dd = as_h2(dv | (dv << 16));
      // -(1024 + z) as an fp16 pair (z is a small non-negative integer held in fp16)
      const __half zh = __hneg(__hadd(__ushort_as_half(static_cast<unsigned short>(zv)), __float2half_rn(1024.0f)));
      const __half2 zz = __halves2half2(zh, zh);
      const int b0 = hb % kABufs, b1 = (hb + 1) % kABufs;
      bool okw = hb < kABufs ||
                 wait_or_abort(&wempty[b0], static_cast<uint32_t>(hb / kABufs - 1) & 1u, abort_flag, a.ws_status);
      okw = okw && (hb + 1 < kABufs || wait_or_abort(&wempty[b1], static_cast<uint32_t>((hb + 1) / kABufs - 1) & 1u,
                                                    abort_flag, a.ws_status));
      if (__any_sync(0xffffffffu, !okw)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        const uint32_t r0 = arow0 + static_cast<uint32_t>(b0 * kABufBytes);
        const uint32_t r1 = arow0 + static_cast<uint32_t>(b1 * kABufBytes);
        const uint32_t cw[4] = {c0.x, c0.y, c0.z, c0.w};
        const uint32_t cv[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t j = static_cast<uint32_t>(4 * p + i);  // word of the half = 16-byte chunk
          sts128(r0 + (((j ^ asw) & 7u) << 4), dq_word(cw[i], zz, dd));
          sts128(r1 + (((j ^ asw) & 7u) << 4), dq_word(cv[i], zz, dd));
        }
        // the MMAs read these rows through the async proxy
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&wfull[b0]);
        mbar_arrive(&wfull[b1]);
      }
      hb += 2;
      // the previous row block's accumulator is complete by now: read it out
      if (pend >= 0) {
        flush(pend, pend_rb, pend_contrib);
        pend = -1;
        if (!ok) break;
      }
      if (i == 0 || g == 0) start = i;
      if (i == cnt - 1 || g == a.Kg - 1) {
        pend = f++;
        pend_rb = u / a.Kg;
        pend_contrib = i - start + 1;
      }
    }
    if (ok && pend >= 0) flush(pend, pend_rb, pend_contrib);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Sums the partial-sum slots of the row blocks no single CTA covered, in CTA
// order (so y does not depend on timing), and writes y.  Block (rb, cy) covers
// the 256 rows of row block rb and tokens 16 cy .. 16 cy + 15; thread (r, j)
// takes row r and tokens 16 cy + 4 j .. + 3.  A thread issues the loads of up
// to kFinBatch contributing CTAs before adding any of them, so the slots cost
// one trip to L2 per batch rather than one per CTA.
constexpr int kFinBatch = 8;
template <int MP>
__global__ void __launch_bounds__(kRows * 4) gemm_tc_finalize(const TcArgs a, int grid_main) {
  // the next layer's main kernel may start its prologue and weight prefetch; it
  // reads x (this kernel's y) only after its own griddepcontrol.wait
  griddep_launch_dependents();
  griddep_wait();
  const int rb = blockIdx.x;
  const int base = a.total_units / grid_main;
  const int rem = a.total_units - base * grid_main;
  const int c0 = owner_cta(rb * a.Kg, base, rem);
  const int c1 = owner_cta(rb * a.Kg + a.Kg - 1, base, rem);
  if (c0 == c1) return;  // one CTA covered the row block and wrote y itself
  const int r = threadIdx.x, cg = blockIdx.y * 4 + threadIdx.y;
  const int n = rb * kRows + r;
  if (n >= a.N || cg >= MP / 4) return;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  for (int cb = c0; cb <= c1; cb += kFinBatch) {
    float4 v[kFinBatch];
#pragma unroll
    for (int j = 0; j < kFinBatch; ++j) {
      const int c = cb + j;
      if (c <= c1) {
        const int rbc = (c * base + min(c, rem)) / a.Kg;  // row block where c's range starts
        v[j] = __ldcg(a.ws_part + static_cast<size_t>(c * 2 + (rb == rbc ? 0 : 1)) * (kRows * MP / 4) + cg * kRows + r);
      }
    }
#pragma unroll
    for (int j = 0; j < kFinBatch; ++j) {
      if (cb + j <= c1) {
        s0 += v[j].x;
        s1 += v[j].y;
        s2 += v[j].z;
        s3 += v[j].w;
      }
    }
  }
  const float sv[4] = {s0, s1, s2, s3};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (cg * 4 + j < a.M) a.y[static_cast<size_t>(cg * 4 + j) * a.N + n] = __float2half_rn(sv[j]);
}

int stages_for(int mp) {
  const int stage = kCodeBytes + 2 * mp * 128;
  int s = (kMaxSmem - 1024 - kCtrlBytes - kABufs * kABufBytes) / stage;
  return s > kMaxStages ? kMaxStages : s;
}

template <int MP>
cudaError_t launch_mp(const TcArgs& a0, const CUtensorMap& tq, const CUtensorMap& tx, int grid, cudaStream_t st) {
  TcArgs a = a0;
  a.stages = stages_for(MP);
  if (a.stages < 2) return cudaErrorNotSupported;
  const int smem = 1024 + a.stages * (kCodeBytes + 2 * MP * 128) + kABufs * kABufBytes + kCtrlBytes;
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(gemm_tc_kernel<MP>),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<MP>, a, tq, tx);
  if (e != cudaSuccess) return e;
  // the partial sums of row blocks shared by several CTAs; asking for the same
  // shared-memory carveout as the main kernel spares the SMs a reconfiguration
  // between the two launches
  e = ensure_func_attr(reinterpret_cast<const void*>(gemm_tc_finalize<MP>), cudaFuncAttributePreferredSharedMemoryCarveout,
                       cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int row_blocks = (a.N + kRows - 1) / kRows;
  cudaLaunchConfig_t fin = {};
  fin.gridDim = dim3(row_blocks, (MP / 4 + 3) / 4);
  fin.blockDim = dim3(kRows, 4);
  fin.stream = st;
  fin.attrs = attr;
  fin.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&fin, gemm_tc_finalize<MP>, a, grid);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The token tile of a launch: M rounded up to 16 up to 64, then 96 or 128.
int tc_tile(int M) {
  const int mp = (M + 15) / 16 * 16;
  return mp <= 64 ? mp : (mp <= 96 ? 96 : 128);
}

}  // namespace

size_t tc_partial_bytes(int M) {
  const size_t mp = static_cast<size_t>(tc_tile(M));
  return 2 * static_cast<size_t>(device_sm_count()) * kRows * mp * 4;
}

cudaError_t launch_gemm_tc(const GemmProblem& p, const Workspace& ws, cudaStream_t st) {
  if (p.M < 1 || p.M > kMaxM || !ws.part) return cudaErrorNotSupported;
  const int mp = tc_tile(p.M);
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;

  // codes: u32 [N][K/8], boxes of 256 rows x 16 words (one group), 64-byte swizzle
  CUtensorMap tq, tx;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.K / 8), static_cast<cuuint64_t>(p.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.K / 8) * 4};
    const cuuint32_t box[2] = {16, static_cast<cuuint32_t>(kRows)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(p.qweight), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // x: fp16 [M][K], boxes of MP rows (rows past M read as zero) x 64 inputs, 128-byte swizzle
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.K), static_cast<cuuint64_t>(p.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.K) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(mp)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(p.x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }

  TcArgs a;
  a.qweight = p.qweight;
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.ws_part = reinterpret_cast<float4*>(ws.part);
  a.ws_status = ws.status;
  a.M = p.M;
  a.N = p.N;
  a.Kw = p.K / 8;
  a.Kg = p.K / kGroup;
  a.dz_w = a.Kg % 8 == 0 ? 8 : (a.Kg % 4 == 0 ? 4 : (a.Kg % 2 == 0 ? 2 : 1));
  const int row_blocks = (p.N + kRows - 1) / kRows;
  a.total_units = row_blocks * a.Kg;
  a.stages = 0;
  const int grid = min(device_sm_count(), a.total_units);
  switch (mp) {
    case 16: return launch_mp<16>(a, tq, tx, grid, st);
    case 32: return launch_mp<32>(a, tq, tx, grid, st);
    case 48: return launch_mp<48>(a, tq, tx, grid, st);
    case 64: return launch_mp<64>(a, tq, tx, grid, st);
    case 96: return launch_mp<96>(a, tq, tx, grid, st);
    default: return launch_mp<128>(a, tq, tx, grid, st);
  }
}

}  // namespace w4a16
