// W4A16 skinny GEMM on the 5th-generation tensor cores (tcgen05), up to 256
// tokens per launch (larger M runs as chunks of 256 tokens, one launch per
// chunk); from 9 tokens, or from 2 where the register-sourced MMA GEMV does not
// apply.
//
//   y[m][n] = sum_k x[m][k] * w_hat[n][k],   w_hat = Delta[n][g] * (u[n][k] - z[n][g])
//
// Once several tokens share each weight, the product is a dense contraction and
// belongs on the tensor cores ("MIT 6.5940 Fall 2024 Lecture 13: LLM
// Deployment" reading guide, §SmoothQuant: batching moves the work from
// memory-bound GEMV towards compute).  Up to M = 64 it is still bound by reading
// the packed weights, so every stage of the kernel is a separate role working
// on its own ring, and the roles overlap: codes stream from HBM, warps turn them
// into w_hat, the tensor cores multiply, and the last tile's sums are read out,
// all at the same time.
//
// Swap-AB.  Weight rows are the MMA's M dimension (a tile of 128 rows = the 128
// lanes of tensor memory) and tokens its N dimension (the token tile MP: 16, 32,
// 64, 96, 128, 192 or 256): D[n][m] = sum_k A[n][k] B[m][k], with A = w_hat in
// tensor memory (fp16 pairs, one 32-bit column per two inputs, written by
// tcgen05.st) and B = x in shared memory (K-major, 128-byte swizzle, rows past M
// zero-filled by the tensor copy), fp32 accumulators in tensor memory.  Keeping
// A out of shared memory leaves shared memory to the copies alone.
//
// Work split (stream-K).  Units are (tile of 128 rows, 4 groups = 512 inputs),
// ordered tile-major and dealt to a persistent grid (one CTA per SM) in
// contiguous, equal ranges.  A CTA's range covers at most a few tiles; it
// accumulates each one (a segment) in a tensor-memory accumulator.  A tile no
// single CTA covers is finished by the lowest CTA that covers part of it (its
// owner), for which the tile is the last segment: every other contributor has
// the tile as its first segment, publishes its fp32 partial tile to a workspace
// slot and adds 1 to its flag per epilogue warp; the owner, after its own MMAs,
// waits for those flags (bounded), adds the partials in CTA order, writes y and
// puts the flags back to 0.  y does not depend on timing, and no second kernel
// is needed.
//
// Roles (24 warps):
//   warp 0       one thread streams the codes: per unit two adjacent tensor
//                copies of 128 rows x 128 bytes (128-byte swizzle, 32 KiB in
//                all) into a ring of Sc stages;
//   warp 1       allocates tensor memory; one thread issues the MMAs (8 of
//                128 x MP x 16 per group, W4A16; 4 of 128 x MP x 32, W4A8) and
//                their commits, waiting on one barrier per unit;
//   warps 2, 3   one thread each streams x, alternating stages: one 3-D tensor
//                copy of a [K / 64][M][64] view per stage (a unit's x up to
//                MP = 32, half of it up to 128, one group above), after
//                griddepcontrol.wait;
//   warps 4-19   dequantization: warp w covers tensor-memory lane quarter w & 3
//                (rows 32 (w & 3) .. + 31 of the tile) and group h = (w - 4) >> 2
//                of each unit; lane i reads its row's 64 code bytes, converts
//                them into w_hat and stores them with tcgen05.st (four warps per
//                lane quarter, so that their latencies overlap);
//   warps 20-23  epilogue: accumulator read-out, y, partial tiles, the owner's sums.
// Dequantization of a code pair: (w >> 4t) & 0x000F000F | 0x64006400 (one LOP3)
// reads as the fp16 pair 1024 + q; subtracting 1024 + z is exact and the
// multiply by Delta rounds once (Lecture 13 guide, §TinyChat, slides 36-37;
// "CMU 11-868 Model Quantization" guide, §BF16/HFMA2).
//
// Every wait is bounded: a timeout sets the workspace status word and an abort
// flag, every role leaves its loop, copies and MMAs in flight are waited for and
// tensor memory is freed before the CTA exits.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

constexpr int kRows = 128;                 // weight rows per tile
constexpr int kCodeStage = kRows * 256;    // 32 KiB: the codes of one unit (4 groups of a tile)
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMaxCodeStages = 8;
constexpr int kMaxXStages = 4;
constexpr int kWarps = 24;
constexpr int kThreads = kWarps * 32;
constexpr int kCodeWarp = 0, kMmaWarp = 1, kXWarp = 2, kXWarp2 = 3;
constexpr int kDqWarp0 = 4, kDqWarps = 16;
constexpr int kDqSets = kDqWarps / 4;   // dequantizing warps per tensor-memory lane quarter
constexpr int kGpw = 4 / kDqSets;       // groups of a unit per dequantizing warp
constexpr int kEpiWarp0 = kDqWarp0 + kDqWarps, kEpiWarps = 4;
constexpr int kCtrlBytes = 1024;
constexpr uint32_t kTmemCols = 512;

struct TcArgs {
  const __half* scales;   // W4A16: Delta and z, fp16 [N][G]
  const __half* zeros;
  const uint8_t* s2;      // W4A8: level-2 step and scaled zero, bytes [N][G]
  const uint8_t* zs;
  const __half* xs;       // W4A8: token scales [M] and channel scales [N]
  const __half* s1;
  int32_t* acc;           // W4A8: optional exact accumulators [M][N]
  __half* y;
  float4* part;           // [grid][MP / 4][128] partial tiles (fp32, or int32 bit patterns)
  uint32_t* flags;        // [grid] partial tile published (left zero after each call)
  uint32_t* status;
  int M, N, G, Q;         // tokens, rows, groups per row, units (4 groups) per row
  int total;              // units = tiles x Q
  int sc, sx;             // code and x ring depths
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

// The MMA issue is warp-collective: the whole warp runs the issue loop with its
// operands the same in every lane, and one elected lane issues each instruction.
// On B200 that issues a 128 x 16 x 16 MMA every 25 cycles, against 50 when a
// single lane runs the loop alone (a one-warp microbenchmark, A in tensor memory).

// D[tmem] (+)= A[tmem] * B[smem]^T: A is 128 rows x 16 inputs (fp16 pairs in 8
// consecutive columns), B is described by a shared-memory matrix descriptor.
// Called by all 32 lanes of the warp with the same arguments.
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

// Arrives once on `bar` when every MMA issued so far by the elected lanes of this
// warp has completed (called by all 32 lanes; one commits).
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns into registers: thread i reads lane (base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (leading offset unused for this layout; encoded as 1).
__device__ __forceinline__ uint64_t sw128_desc(const void* p) {
  const uint32_t a = smem_u32(p);
  const uint32_t lo = ((a >> 4) & 0x3FFFu) | (1u << 16);
  const uint32_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// kind::f16 instruction descriptor: fp32 D, fp16 A and B, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// ---- waits, arrivals -------------------------------------------------------------
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

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Waits (bounded) until a partial-tile flag reaches `want`.
__device__ __forceinline__ bool wait_flag(const uint32_t* flag, uint32_t want, volatile uint32_t* abort_flag,
                                          uint32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (ld_acquire(flag) >= want) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, kDevWaitTimeout);
      return false;
    }
    __nanosleep(64);
  }
}

__device__ __forceinline__ uint32_t lop3_nib(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
  return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint16_t ld_nc_u16(const __half* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// (1024 + u) - (1024 + z) = u - z exactly, computed as an FMA with 1 (the fp16
// add and subtract instructions issue far slower than FMA on sm_100a), then one
// rounding in the multiply by Delta.  nz = -(1024 + z).
__device__ __forceinline__ uint32_t dq_pair(uint32_t v, __half2 nz, __half2 dd) {
  return as_u32(__hmul2(__hfma2(as_h2(lop3_nib(v)), __float2half2_rn(1.0f), nz), dd));
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---- the two arithmetics ------------------------------------------------------
// W4A16: A = w_hat fp16 (one 32-bit column per two inputs: 64 columns per
// group), B = x fp16 (a 128-byte chunk of a token row holds 64 inputs: two
// chunks per group), kind::f16 MMAs of K = 16, fp32 accumulators.
// W4A8 ("MIT 6.5940 Fall 2024 Lecture 13" reading guide, §QServe): A = w8_hat =
// u * s2 - zs int8 (one column per four inputs: 32 per group), B = x8 int8 (one
// chunk per group), kind::i8 MMAs of K = 32, exact int32 accumulators.
// Either way an MMA reads 32 bytes of each A and B row (8 columns of A, one
// 32-byte step of the B descriptor), and a group is four MMAs per chunk.
template <bool I8>
struct Arith {
  static constexpr int kACols = I8 ? 32 : 64;          // tensor-memory columns of A per group
  static constexpr int kChunks = I8 ? 1 : 2;           // 128-byte x chunks per group (4 MMAs each)
};

// kind::i8 instruction descriptor: s32 D, signed 8-bit A and B, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_i8_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

__device__ __forceinline__ uint16_t ld_nc_b8(const uint8_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// Bytewise a - b modulo 256 in each of the four bytes (no borrow between bytes):
// (a | 0x80) - (b & 0x7F) cannot borrow, and the top bit is then fixed up.
__device__ __forceinline__ uint32_t sub_bytes(uint32_t a, uint32_t b_low7, uint32_t b_top_not) {
  return ((a | 0x80808080u) - b_low7) ^ ((a & 0x80808080u) ^ b_top_not);
}

// W4A8 level-2 dequantization of one code word (inputs 8j .. 8j + 7): two
// columns of four int8 values each, inputs in order.  Layout v1 puts element i
// in nibble slot [0,4,1,5,2,6,3,7][i]: w & 0x0F0F0F0F holds elements 0,4,1,5
// in its bytes and (w >> 4) & 0x0F0F0F0F elements 2,6,3,7.  One multiply per
// four codes applies s2 (u * s2 <= 240 fits a byte, so no carries) before the
// zero point is subtracted byte by byte (the progressive order).
__device__ __forceinline__ void dq8_word(uint32_t w, uint32_t s2, uint32_t zlo7, uint32_t ztop, uint32_t& c0,
                                         uint32_t& c1) {
  const uint32_t lo = sub_bytes((w & 0x0F0F0F0Fu) * s2, zlo7, ztop);
  const uint32_t hi = sub_bytes(((w >> 4) & 0x0F0F0F0Fu) * s2, zlo7, ztop);
  c0 = __byte_perm(lo, hi, 0x6420);  // elements 0, 1, 2, 3
  c1 = __byte_perm(lo, hi, 0x7531);  // elements 4, 5, 6, 7
}

// Accumulator buffers: two (double-buffered across segments) up to MP = 128, one
// above.  The w_hat slots (one group each) take the columns from kACol0 up.
__host__ __device__ constexpr int n_acc(int mp) { return mp <= 128 ? 2 : 1; }
template <bool I8>
__host__ __device__ constexpr int n_aslots(int mp) {
  return (512 - n_acc(mp) * mp) / Arith<I8>::kACols > 8 ? 8 : (512 - n_acc(mp) * mp) / Arith<I8>::kACols;
}
// Groups of x per x stage: the x of a whole unit up to MP = 32, half of it up
// to 128, one group above.
__host__ __device__ constexpr int x_groups(int mp) { return mp <= 32 ? 4 : (mp <= 128 ? 2 : 1); }

// Unit u of the range partition: the CTA whose range holds it.
__host__ __device__ __forceinline__ int owner_cta(int u, int base, int rem) {
  const int big = rem * (base + 1);
  return u < big ? u / (base + 1) : rem + (u - big) / base;
}

template <int MP, bool I8>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tx) {
  using AR = Arith<I8>;
  constexpr int kXG = x_groups(MP);                           // groups per x stage
  // With at most two x stages per unit (MP <= 128; the ring holds at least two)
  // the dequantizing warps wait for a unit's x before they release its w_hat,
  // so the MMA thread waits on one barrier per unit.  Above, a unit's four x
  // stages do not fit the ring at once and the MMA thread waits for each.
  constexpr bool kXByDq = 4 / kXG <= 2;
  constexpr int kXChunk = MP * 128;                           // one 128-byte chunk of every token
  constexpr int kXStage = kXG * AR::kChunks * kXChunk;
  constexpr uint32_t kIdesc = I8 ? idesc_i8(MP) : idesc_f16(MP);
  constexpr int kAcc = n_acc(MP);
  constexpr int kASlots = n_aslots<I8>(MP);
  constexpr uint32_t kACol0 = kTmemCols - static_cast<uint32_t>(AR::kACols * kASlots);
  static_assert(kAcc * MP <= static_cast<int>(kACol0), "accumulators and w_hat slots exceed tensor memory");
  static_assert(kASlots >= 4, "w_hat needs a unit's worth of slots");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Sc = a.sc, Sx = a.sx;
  uint8_t* cstage = smem;                                  // Sc x 32 KiB of codes
  uint8_t* xstage = cstage + Sc * kCodeStage;              // Sx x kXStage of x
  uint64_t* bars = reinterpret_cast<uint64_t*>(xstage + Sx * kXStage);
  uint64_t* cfull = bars;                                  // [Sc] codes landed
  uint64_t* cempty = cfull + kMaxCodeStages;               // [Sc] codes read
  uint64_t* xfull = cempty + kMaxCodeStages;               // [Sx] x landed
  uint64_t* xempty = xfull + kMaxXStages;                  // [Sx] x consumed by the MMAs
  uint64_t* afull = xempty + kMaxXStages;                  // [2] w_hat of a unit written (units alternate)
  uint64_t* aempty = afull + 8;                            // [kASlots] w_hat of a group consumed
  uint64_t* accfull = aempty + 8;                          // [kAcc] segment's MMAs complete
  uint64_t* accempty = accfull + 2;                        // [kAcc] accumulator read out
  uint64_t* tdown = accempty + 2;                          // teardown: all MMAs complete
  uint32_t* tslot = reinterpret_cast<uint32_t*>(tdown + 1);
  volatile uint32_t* abort_flag = tslot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grid = static_cast<int>(gridDim.x), bx = static_cast<int>(blockIdx.x);
  const int base = a.total / grid, rem = a.total - base * grid;
  const int u0 = bx * base + min(bx, rem);
  const int cnt = base + (bx < rem ? 1 : 0);
  const int Q = a.Q;
  const int xper = 4 / kXG;  // x stages per unit

  if (threadIdx.x == 0) {
    for (int s = 0; s < Sc; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], kDqWarps);
    }
    for (int s = 0; s < Sx; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&afull[b], kDqWarps);  // a unit's w_hat, alternate units
    for (int b = 0; b < kASlots; ++b) mbar_init(&aempty[b], 1);
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], kEpiWarps);
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
  // the next kernel on the stream may begin its prologue (it waits for this
  // grid's completion before it reads y or reuses the workspace)
  griddep_launch_dependents();

  if (warp == kCodeWarp) {
    // ---------------- codes: two adjacent 16 KiB boxes per unit ----------------
    if (lane == 0) {
      prefetch_tensor_map(&tq);
      const uint64_t pol = l2_evict_first_policy();
      int issued = 0;
      // the weights do not depend on the previous kernel: no griddepcontrol.wait
      for (int i = 0; i < cnt; ++i) {
        const int s = i % Sc;
        if (i >= Sc && !wait_or_abort(&cempty[s], static_cast<uint32_t>(i / Sc - 1) & 1u, abort_flag, a.status))
          break;
        const int u = u0 + i, t = u / Q, q4 = u - t * Q;
        uint8_t* dst = cstage + s * kCodeStage;
        mbar_arrive_expect_tx(&cfull[s], kCodeStage);
        tma_load_2d(dst, &tq, q4 * 64, t * kRows, &cfull[s], pol);
        tma_load_2d(dst + kCodeStage / 2, &tq, q4 * 64 + 32, t * kRows, &cfull[s], pol);
        issued = i + 1;
      }
      // After an abort the copies in flight must land before the CTA may exit
      // (otherwise every stage was consumed): the last Sc issues, one per stage.
      if (*abort_flag)
        for (int j = max(0, issued - Sc); j < issued; ++j)
          mbar_wait_bounded(&cfull[j % Sc], static_cast<uint32_t>(j / Sc) & 1u);
    }
  } else if (warp == kXWarp || warp == kXWarp2) {
    // ---------------- x: one 3-D box per stage; the two x warps alternate stages ----------------
    if (lane == 0) {
      prefetch_tensor_map(&tx);
      const uint64_t pol = l2_evict_last_policy();
      griddep_wait();  // x may be the previous kernel's output
      const int total_x = cnt * xper;
      int latest[kMaxXStages];  // this warp's latest issue into each stage
#pragma unroll
      for (int s = 0; s < kMaxXStages; ++s) latest[s] = -1;
      for (int j = (warp == kXWarp ? 0 : 1); j < total_x; j += 2) {
        const int s = j % Sx;
        if (j >= Sx && !wait_or_abort(&xempty[s], static_cast<uint32_t>(j / Sx - 1) & 1u, abort_flag, a.status))
          break;
        const int i = j / xper, u = u0 + i, q4 = u % Q;
        const int g0 = 4 * q4 + (j - i * xper) * kXG;  // first group of the stage
        mbar_arrive_expect_tx(&xfull[s], kXStage);
        tma_load_3d(xstage + s * kXStage, &tx, 0, 0, g0 * AR::kChunks, &xfull[s], pol);
        latest[s] = j;
      }
      // after an abort, this warp's copies in flight land before the CTA may exit
      if (*abort_flag)
        for (int s = 0; s < Sx; ++s)
          if (latest[s] >= 0) mbar_wait_bounded(&xfull[s], static_cast<uint32_t>(latest[s] / Sx) & 1u);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer (the whole warp; one lane issues) ----------------
    // A wait on an mbarrier between MMAs costs about as much as 5 MMAs of
    // 128 x 16 x 16 (B200 measurement), even when the phase is already complete,
    // so w_hat is signalled per unit (32 MMAs), not per group.  Every lane waits
    // and the outcome is agreed on by the warp, so the lanes stay converged.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag, a.status));
    };
    bool any = false, ok = true;
    int seg = 0;
    for (int i = 0; i < cnt && ok; ++i) {
      const int u = u0 + i, q4 = u % Q;
      const bool first = (i == 0) || (q4 == 0);
      const bool last = (i == cnt - 1) || (q4 == Q - 1);
      const int ab = seg % kAcc;
      if (first && seg >= kAcc && !wait_all(&accempty[ab], static_cast<uint32_t>(seg / kAcc - 1) & 1u)) break;
      const uint32_t d = tbase + static_cast<uint32_t>(ab * MP);
      // the unit's w_hat (all four groups) is in tensor memory (and, when kXByDq,
      // its x stages have landed: the dequantizing warps wait for those first)
      if (!wait_all(&afull[i & 1], static_cast<uint32_t>(i >> 1) & 1u)) break;
      tc_fence_after();
      for (int gg = 0; gg < 4; ++gg) {
        const int j = i * xper + gg / kXG;  // x stage of this group
        const int s = j % Sx;
        if (!kXByDq && gg % kXG == 0 && !wait_all(&xfull[s], static_cast<uint32_t>(j / Sx) & 1u)) {
          ok = false;
          break;
        }
        // every group position of a unit takes its w_hat slot, a position past the
        // last group (K / 128 not a multiple of 4) with no MMAs, so that each slot's
        // uses follow one another in order
        const int ga = 4 * i + gg, b = ga % kASlots;
        if (4 * q4 + gg < a.G) {
          const uint32_t acol = tbase + kACol0 + static_cast<uint32_t>(b * AR::kACols);
          const uint8_t* xg = xstage + s * kXStage + (gg % kXG) * AR::kChunks * kXChunk;
#pragma unroll
          for (int c = 0; c < AR::kChunks; ++c) {
            const uint64_t bd = sw128_desc(xg + c * kXChunk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // the descriptor's start address advances 32 bytes (2 x 16) per MMA
              const uint32_t at = acol + 8u * (4 * c + kk);
              const bool accum = !(first && gg == 0 && c == 0 && kk == 0);
              if constexpr (I8)
                mma_i8_ts(d, at, bd + 2u * kk, kIdesc, accum);
              else
                mma_f16_ts(d, at, bd + 2u * kk, kIdesc, accum);
            }
          }
          any = true;
        }
        mma_commit(&aempty[b]);
        if (gg % kXG == kXG - 1) mma_commit(&xempty[s]);
      }
      if (!ok) break;
      if (last) {
        mma_commit(&accfull[ab]);
        ++seg;
      }
    }
    if (any) {
      mma_commit(tdown);
      mbar_wait_bounded(tdown, 0);
    }
  } else if (warp >= kDqWarp0 && warp < kDqWarp0 + kDqWarps) {
    // ---------------- dequantization into tensor memory ----------------
    // warp (q, h): rows 32 q .. 32 q + 31 of the tile, groups h + kDqSets e of each unit
    const int q = warp & 3, h = (warp - kDqWarp0) >> 2;
    const int r = q * 32 + lane;  // row within the tile
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(q * 32) << 16) + kACol0;
    const uint32_t rsw = static_cast<uint32_t>(r & 7);
    // Per-group parameters, fetched two units ahead into one of two register
    // sets (even and odd units): a value is first read two units after its load
    // was issued, so the load's latency (HBM, under the code stream) is hidden.
    // (A look-ahead by shifting a register array reads each value one unit after
    // its load: every shift waits for the previous unit's load.)
    uint16_t pd[2][kGpw], pz[2][kGpw];
    auto fetch = [&](int it, uint16_t& dv, uint16_t& zv) {
      dv = zv = 0;
      const int i = it / kGpw;
      if (i < cnt) {
        const int u = u0 + i, t = u / Q, g = 4 * (u - t * Q) + h + kDqSets * (it % kGpw);
        const int n = t * kRows + r;
        if (n < a.N && g < a.G) {
          const size_t o = static_cast<size_t>(n) * a.G + g;
          if constexpr (I8) {
            dv = ld_nc_b8(a.s2 + o);
            zv = ld_nc_b8(a.zs + o);
          } else {
            dv = ld_nc_u16(a.scales + o);
            zv = ld_nc_u16(a.zeros + o);
          }
        }
      }
    };
#pragma unroll
    for (int par = 0; par < 2; ++par)
#pragma unroll
      for (int e = 0; e < kGpw; ++e) fetch(kGpw * par + e, pd[par][e], pz[par][e]);
    bool ok = true;
    for (int i2 = 0; i2 < cnt && ok; i2 += 2)
#pragma unroll
    for (int par = 0; par < 2; ++par) {
      const int i = i2 + par;
      if (i >= cnt || !ok) break;
      const int u = u0 + i, t = u / Q, q4 = u - t * Q;
      const int s = i % Sc;
      const bool okc = wait_or_abort(&cfull[s], static_cast<uint32_t>(i / Sc) & 1u, abort_flag, a.status);
      if (__any_sync(0xffffffffu, !okc)) {
        ok = false;
        break;
      }
      // this lane's 64 code bytes of each of its groups gg (the pair box gg / 2, half gg % 2)
      uint4 cw[kGpw][4];
      bool valid[kGpw];
#pragma unroll
      for (int e = 0; e < kGpw; ++e) {
        const int gg = h + kDqSets * e;
        valid[e] = 4 * q4 + gg < a.G;
        if (valid[e]) {
          const uint32_t row = smem_u32(cstage) + static_cast<uint32_t>(s * kCodeStage + (gg >> 1) * (kCodeStage / 2) + r * 128);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            cw[e][c] = lds128(row + (((static_cast<uint32_t>(4 * (gg & 1) + c)) ^ rsw) << 4));
        }
      }
      // every lane's reads are ordered before the copy that refills the stage
      release_stage_reads();
      __syncwarp();
      if (lane == 0) mbar_arrive(&cempty[s]);
#pragma unroll
      for (int e = 0; e < kGpw; ++e) {
        const int gg = h + kDqSets * e;
        const uint16_t dv = pd[par][e], zv = pz[par][e];
        fetch(kGpw * (i + 2) + e, pd[par][e], pz[par][e]);
        const int ga = 4 * i + gg, b = ga % kASlots;
        // Each of this warp's slots of the unit must be free.  The MMA warp
        // commits the slots in group order and a commit arrives only once every
        // earlier MMA has completed, so the wait for the warp's last slot of the
        // unit covers all: one barrier wait per unit (each costs hundreds of cycles).
        if (e == 0) {
          const int gl = ga + kDqSets * (kGpw - 1);
          const bool oka = gl < kASlots || wait_or_abort(&aempty[gl % kASlots], static_cast<uint32_t>(gl / kASlots - 1) & 1u,
                                                         abort_flag, a.status);
          if (__any_sync(0xffffffffu, !oka)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        const uint32_t col = lane_base + static_cast<uint32_t>(b * AR::kACols);
        // a position past the last group writes no w_hat, but its slot is taken in turn
        if (!valid[e]) continue;  // uniform over the warp
        if constexpr (I8) {
          const uint32_t s2 = dv, zs4 = static_cast<uint32_t>(zv) * 0x01010101u;
          const uint32_t zlo7 = zs4 & 0x7F7F7F7Fu, ztop = ~zs4 & 0x80808080u;
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int k = 0; k < 4; ++k) dq8_word((&cw[e][c].x)[k], s2, zlo7, ztop, v[8 * c + 2 * k], v[8 * c + 2 * k + 1]);
          tmem_st32(col, v);
        } else {
          const __half2 dd = as_h2(static_cast<uint32_t>(dv) | (static_cast<uint32_t>(dv) << 16));
          // -(1024 + z) as an fp16 pair (z is a small non-negative integer held in fp16)
          const __half zh = __hneg(__hadd(__ushort_as_half(zv), __float2half_rn(1024.0f)));
          const __half2 nz = __halves2half2(zh, zh);
#pragma unroll
          for (int c = 0; c < 4; c += 2) {
            uint32_t v[32];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const uint32_t wv[4] = {cw[e][c + h2].x, cw[e][c + h2].y, cw[e][c + h2].z, cw[e][c + h2].w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                v[16 * h2 + 4 * k + 0] = dq_pair(wv[k], nz, dd);
                v[16 * h2 + 4 * k + 1] = dq_pair(wv[k] >> 4, nz, dd);
                v[16 * h2 + 4 * k + 2] = dq_pair(wv[k] >> 8, nz, dd);
                v[16 * h2 + 4 * k + 3] = dq_pair(wv[k] >> 12, nz, dd);
              }
            }
            tmem_st32(col + static_cast<uint32_t>(16 * c), v);
          }
        }
      }
      if (!ok) break;
      // the unit's x stages must have landed before the MMAs are released (the MMA
      // thread then waits on one barrier per unit); one warp's wait is enough, as
      // the barrier completes only with every warp's arrival
      bool okx = true;
      for (int jx = i * xper; kXByDq && warp == kDqWarp0 && jx < (i + 1) * xper && okx; ++jx)
        okx = wait_or_abort(&xfull[jx % Sx], static_cast<uint32_t>(jx / Sx) & 1u, abort_flag, a.status);
      if (__any_sync(0xffffffffu, !okx)) {
        ok = false;
        break;
      }
      // both of this warp's groups of the unit are in tensor memory
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[i & 1]);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(q * 32) << 16);
    griddep_wait();  // y and the workspace slots may still be in use by the previous kernel
    int seg = 0;
    for (int i = 0; i < cnt; ++i) {
      const int u = u0 + i, t = u / Q, q4 = u - t * Q;
      if (!(i == cnt - 1 || q4 == Q - 1)) continue;  // only at the end of a segment
      const int ia = (seg == 0) ? 0 : i - q4;        // segment start (a later segment starts at q4 = 0)
      const bool covers_first = (u0 + ia) == t * Q;
      const bool covers_last = (q4 == Q - 1);
      const int ab = seg % kAcc;
      const bool okw = wait_or_abort(&accfull[ab], static_cast<uint32_t>(seg / kAcc) & 1u, abort_flag, a.status);
      if (__any_sync(0xffffffffu, !okw)) break;
      tc_fence_after();
      const int n = t * kRows + r;
      const uint32_t acc = lane_base + static_cast<uint32_t>(ab * MP);
      bool okw2 = true;
      if (!covers_first) {
        // a contributor: publish the partial tile; each epilogue warp adds 1 to
        // the CTA's flag once its rows are stored, so 4 means the tile is complete
        float4* slot = a.part + static_cast<size_t>(bx) * (MP / 4) * kRows;
#pragma unroll 1
        for (int c = 0; c < MP / 16; ++c) {
          float v[16];
          tmem_ld16(acc + static_cast<uint32_t>(16 * c), v);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            slot[(4 * c + e) * kRows + r] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        }
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(a.flags + bx, 1u);
        }
      } else {
        // alone, or the owner: add the later contributors' partial tiles in CTA order
        const int c_hi = covers_last ? bx : owner_cta(t * Q + Q - 1, base, rem);
        for (int cc = bx + 1; cc <= c_hi && okw2; ++cc) {
          bool okf = true;
          if (lane == 0) okf = wait_flag(a.flags + cc, kEpiWarps, abort_flag, a.status);
          okw2 = __shfl_sync(0xffffffffu, okf, 0);
          if (okw2) (void)ld_acquire(a.flags + cc);  // every lane acquires what the publisher released
        }
        if (okw2) {
          const double s1n = I8 && n < a.N ? static_cast<double>(__half2float(a.s1[n])) : 0.0;
#pragma unroll 1
          for (int c = 0; c < MP / 16; ++c) {
            float v[16];
            tmem_ld16(acc + static_cast<uint32_t>(16 * c), v);
            for (int cc = bx + 1; cc <= c_hi; ++cc) {
              const float4* slot = a.part + static_cast<size_t>(cc) * (MP / 4) * kRows;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float4 w = __ldcg(slot + (4 * c + e) * kRows + r);
                if constexpr (I8) {
                  // the int32 sums travel as their bit patterns; integer addition is exact
                  v[4 * e] = __int_as_float(__float_as_int(v[4 * e]) + __float_as_int(w.x));
                  v[4 * e + 1] = __int_as_float(__float_as_int(v[4 * e + 1]) + __float_as_int(w.y));
                  v[4 * e + 2] = __int_as_float(__float_as_int(v[4 * e + 2]) + __float_as_int(w.z));
                  v[4 * e + 3] = __int_as_float(__float_as_int(v[4 * e + 3]) + __float_as_int(w.w));
                } else {
                  v[4 * e] += w.x;
                  v[4 * e + 1] += w.y;
                  v[4 * e + 2] += w.z;
                  v[4 * e + 3] += w.w;
                }
              }
            }
            if (n < a.N) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int m = 16 * c + e;
                if (m >= a.M) continue;
                if constexpr (I8) {
                  const int iv = __float_as_int(v[e]);
                  const double yv = (static_cast<double>(iv) * static_cast<double>(__half2float(a.xs[m]))) * s1n;
                  uint16_t hb;
                  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(hb) : "d"(yv));
                  a.y[static_cast<size_t>(m) * a.N + n] = __ushort_as_half(hb);
                  if (a.acc) a.acc[static_cast<size_t>(m) * a.N + n] = iv;
                } else {
                  a.y[static_cast<size_t>(m) * a.N + n] = __float2half_rn(v[e]);
                }
              }
            }
          }
          // Each owner warp adds 1 once it has read a flag's tile; the last of
          // the four (seeing 2 x 4 - 1) puts the flag back to zero for the next
          // call, which starts only after this grid has ended.
          __syncwarp();
          if (lane == 0)
            for (int cc = bx + 1; cc <= c_hi; ++cc)
              if (atomicAdd(a.flags + cc, 1u) == 2 * kEpiWarps - 1) atomicExch(a.flags + cc, 0u);
        }
      }
      if (!okw2) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[ab]);
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Ring depths: x stages for two units of x when that fits in 128 KiB (so that
// the x of the next unit can land while the MMAs work on this one), else two
// stages; the rest of shared memory for code stages (at most kMaxCodeStages).
template <int MP, bool I8>
void ring_depths(int& sc, int& sx) {
  const int xs = x_groups(MP) * Arith<I8>::kChunks * MP * 128;
  const int xper = 4 / x_groups(MP);
  sx = 2 * xper * xs <= 128 * 1024 ? 2 * xper : 2;
  sx = sx > kMaxXStages ? kMaxXStages : sx;
  sc = (kMaxSmem - 1024 - kCtrlBytes - sx * xs) / kCodeStage;
  sc = sc > kMaxCodeStages ? kMaxCodeStages : sc;
}

template <int MP, bool I8>
cudaError_t launch_mp(const TcArgs& a0, const CUtensorMap& tq, const CUtensorMap& tx, int grid, cudaStream_t st) {
  TcArgs a = a0;
  ring_depths<MP, I8>(a.sc, a.sx);
  if (a.sc < 2) return cudaErrorNotSupported;
  const int smem = 1024 + a.sc * kCodeStage + a.sx * x_groups(MP) * Arith<I8>::kChunks * MP * 128 + kCtrlBytes;
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(gemm_tc_kernel<MP, I8>),
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
  e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<MP, I8>, a, tq, tx);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The token tile of a launch of M <= kMaxM tokens.
int tc_tile(int M) {
  const int mp = (M + 15) / 16 * 16;
  if (mp <= 32) return mp <= 16 ? 16 : 32;
  if (mp <= 64) return 64;
  if (mp <= 96) return 96;
  if (mp <= 128) return 128;
  return mp <= 192 ? 192 : 256;
}

// Tensor maps of a launch: codes u32 [N][K/8] in boxes of 128 rows x 32 words
// (one pair of groups; a unit takes two), and x as a 3-D view [K / E][M][E]
// (E = 64 fp16 or 128 int8: one 128-byte chunk) in boxes of E x MP x the
// chunks of one x stage, all with the 128-byte swizzle.
bool encode_maps(const uint32_t* qweight, const void* x, bool i8, int M, int N, int K, int mp, CUtensorMap& tq,
                 CUtensorMap& tx) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 8), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 8) * 4};
    const cuuint32_t box[2] = {32, static_cast<cuuint32_t>(kRows)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(qweight), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    const int elem = i8 ? 1 : 2, E = 128 / elem;
    const int chunks_per_stage = x_groups(mp) * (i8 ? 1 : 2);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(E), static_cast<cuuint64_t>(M),
                                static_cast<cuuint64_t>(K / E)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * elem, 128};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(E), static_cast<cuuint32_t>(mp),
                               static_cast<cuuint32_t>(chunks_per_stage)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tx, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(x), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

template <bool I8>
cudaError_t launch_tc(TcArgs& a, const uint32_t* qweight, const void* x, int K, cudaStream_t st) {
  const int mp = tc_tile(a.M);
  CUtensorMap tq, tx;
  if (!encode_maps(qweight, x, I8, a.M, a.N, K, mp, tq, tx)) return cudaErrorInvalidValue;
  a.G = K / kGroup;
  a.Q = (a.G + 3) / 4;
  const int tiles = (a.N + kRows - 1) / kRows;
  a.total = tiles * a.Q;
  a.sc = a.sx = 0;
  const int grid = min(device_sm_count(), a.total);
  if (grid > kMaxFlags) return cudaErrorNotSupported;
  switch (mp) {
    case 16: return launch_mp<16, I8>(a, tq, tx, grid, st);
    case 32: return launch_mp<32, I8>(a, tq, tx, grid, st);
    case 64: return launch_mp<64, I8>(a, tq, tx, grid, st);
    case 96: return launch_mp<96, I8>(a, tq, tx, grid, st);
    case 128: return launch_mp<128, I8>(a, tq, tx, grid, st);
    case 192: return launch_mp<192, I8>(a, tq, tx, grid, st);
    default: return launch_mp<256, I8>(a, tq, tx, grid, st);
  }
}

}  // namespace

size_t tc_partial_bytes(int M) {
  const size_t mp = static_cast<size_t>(tc_tile(M));
  return static_cast<size_t>(device_sm_count()) * kRows * mp * 4;
}

cudaError_t launch_gemm_tc(const GemmProblem& p, const Workspace& ws, cudaStream_t st) {
  if (p.M < 1 || p.M > kMaxM || !ws.part || !ws.flags) return cudaErrorNotSupported;
  TcArgs a = {};
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.part = reinterpret_cast<float4*>(ws.part);
  a.flags = ws.flags;
  a.status = ws.status;
  a.M = p.M;
  a.N = p.N;
  return launch_tc<false>(a, p.qweight, p.x, p.K, st);
}

cudaError_t launch_w4a8_gemm_tc(const W4A8Problem& p, const Workspace& ws, cudaStream_t st) {
  if (p.M < 1 || p.M > kMaxM || !ws.part || !ws.flags) return cudaErrorNotSupported;
  TcArgs a = {};
  a.s2 = p.s2;
  a.zs = p.zs;
  a.xs = p.sx;
  a.s1 = p.s1;
  a.acc = p.acc;
  a.y = p.y;
  a.part = reinterpret_cast<float4*>(ws.part);
  a.flags = ws.flags;
  a.status = ws.status;
  a.M = p.M;
  a.N = p.N;
  return launch_tc<true>(a, p.qweight, p.x8, p.K, st);
}

}  // namespace w4a16
