// W4A16 skinny GEMM on the 5th-generation tensor cores (tcgen05) for M = 5..64.
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
// tokens its N dimension (MP = M rounded up to 16): D[n][m] = sum_k A[n][k] B[m][k]
// with A = w_hat (fp16, K-major) and B = x (fp16, K-major), fp32 accumulators in
// tensor memory (TMEM lane = weight row, column = token).
//
// Work split.  Units are (row block of 256 rows, group of 128 inputs), ordered
// row-block-major and dealt to a persistent grid (one CTA per SM) in contiguous,
// equal ranges.  A CTA accumulates its units of one row block in two 128 x MP
// TMEM accumulators (double-buffered, so the next row block's MMAs overlap the
// epilogue of the last).  A CTA that covers a whole row block writes y directly;
// otherwise its fp32 partials are added into the workspace and the last
// contributor of the row block converts them to fp16 and zeroes the workspace.
//
// Roles (16 warps):
//   warp 0     one thread issues the tensor copies (TMA) of each unit into a ring
//              of stages: the 256 x 16-word code tile (64-byte swizzle) and the
//              two 64-input halves of the x tile (128-byte swizzle, rows past M
//              zero-filled);
//   warp 1     allocates TMEM; one thread issues tcgen05.mma (8 per 64-input half)
//              and tcgen05.commit;
//   warps 4-7  epilogue: tcgen05.ld of the accumulators, y or workspace;
//   warps 8-15 dequantization: thread r owns weight row r of the block and turns
//              its codes into w_hat in a 128-byte-swizzled K-major tile, the
//              layout the MMA's shared-memory descriptor reads.
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

constexpr int kThreads = 512;
constexpr int kRows = 256;                      // weight rows per row block (two MMA tiles)
constexpr int kCodeBytes = kRows * 16 * 4;      // 16 KiB: one group of codes for the block
constexpr int kWBytes = kRows * 64 * 2;         // 32 KiB: w_hat for 64 inputs of the block
constexpr int kMaxSmem = 227 * 1024;
constexpr int kMaxStages = 8;
constexpr int kCtrlBytes = 256;

struct TcArgs {
  const __half* scales;
  const __half* zeros;
  __half* y;
  float* ws_acc;        // [N][MP]
  uint32_t* ws_cnt;     // [row blocks]
  uint32_t* ws_status;
  int M, N, Kg;
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

// D[tmem] (+)= A[smem] * B[smem]^T, fp16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

// Arrives once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i gets lane (base + i), columns c..c+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
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

// Named barrier over the four epilogue warps; returns the OR of `pred` over them.
__device__ __forceinline__ bool epi_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t lop3_nib(uint32_t w) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
  return r;
}

__device__ __forceinline__ uint32_t ld_nc_u16(const __half* p) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t dq_pair(uint32_t v, __half2 zz, __half2 dd) {
  return as_u32(__hmul2(__hsub2(as_h2(lop3_nib(v)), zz), dd));
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

template <int MP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tx) {
  constexpr int kXHalf = MP * 128;                // one 64-input half of the x tile
  constexpr int kStageBytes = kCodeBytes + 2 * kXHalf;
  constexpr uint32_t kCols = 4 * MP <= 32 ? 32 : (4 * MP <= 64 ? 64 : (4 * MP <= 128 ? 128 : 256));
  constexpr uint32_t kIdesc = idesc_f16(MP);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = a.stages;
  uint8_t* wbuf = smem;                          // 2 x kWBytes
  uint8_t* stages = smem + 2 * kWBytes;          // S x kStageBytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(stages + S * kStageBytes);
  uint64_t* full = bars;                         // [S] codes + x landed
  uint64_t* rempty = bars + kMaxStages;          // [S] codes read, x consumed
  uint64_t* wfull = bars + 2 * kMaxStages;       // [2] w_hat half written
  uint64_t* wempty = wfull + 2;                  // [2] w_hat half consumed by the MMAs
  uint64_t* afull = wfull + 4;                   // [2] accumulator complete
  uint64_t* aempty = wfull + 6;                  // [2] accumulator read out
  uint64_t* tdown = wfull + 8;                   // teardown: all MMAs complete
  uint32_t* tslot = reinterpret_cast<uint32_t*>(wfull + 9);
  volatile uint32_t* abort_flag = tslot + 1;
  volatile uint32_t* last_flag = tslot + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int base = a.total_units / static_cast<int>(gridDim.x);
  const int rem = a.total_units - base * static_cast<int>(gridDim.x);
  const int bx = static_cast<int>(blockIdx.x);
  const int u0 = bx * base + min(bx, rem);
  const int cnt = base + (bx < rem ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&rempty[s], 9);  // 8 dequantization warps + 1 MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&wfull[b], 8);
      mbar_init(&wempty[b], 1);
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], 4);
    }
    mbar_init(tdown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    // ---------------- producer: tensor copies of codes and x ----------------
    if (lane == 0) {
      const uint64_t pol_q = l2_evict_first_policy();
      const uint64_t pol_x = l2_evict_last_policy();
      int issued = 0;
      for (int i = 0; i < cnt; ++i) {
        const int s = i % S;
        if (i >= S && !wait_or_abort(&rempty[s], static_cast<uint32_t>(i / S - 1) & 1u, abort_flag, a.ws_status))
          break;
        const int u = u0 + i, rb = u / a.Kg, g = u - rb * a.Kg;
        uint8_t* st = stages + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(st, &tq, g * 16, rb * kRows, &full[s], pol_q);
        tma_load_2d(st + kCodeBytes, &tx, g * 128, 0, &full[s], pol_x);
        tma_load_2d(st + kCodeBytes + kXHalf, &tx, g * 128 + 64, 0, &full[s], pol_x);
        issued = i + 1;
      }
      // copies still in flight must land before the CTA may exit
      for (int j = max(0, issued - S); j < issued; ++j)
        mbar_wait_bounded(&full[j % S], static_cast<uint32_t>(j / S) & 1u);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool any = false;
      int hb = 0, f = 0;
      for (int i = 0; i < cnt; ++i) {
        const int s = i % S;
        const int u = u0 + i, rb = u / a.Kg, g = u - rb * a.Kg;
        (void)rb;
        const bool first = (i == 0) || (g == 0);
        const bool last = (i == cnt - 1) || (g == a.Kg - 1);
        const int ab = f & 1;
        if (first && f >= 2 && !wait_or_abort(&aempty[ab], static_cast<uint32_t>(f / 2 - 1) & 1u, abort_flag, a.ws_status))
          break;
        if (!wait_or_abort(&full[s], static_cast<uint32_t>(i / S) & 1u, abort_flag, a.ws_status)) break;
        bool ok = true;
        const uint8_t* xs = stages + s * kStageBytes + kCodeBytes;
        for (int h = 0; h < 2; ++h) {
          const int b = hb & 1;
          if (!wait_or_abort(&wfull[b], static_cast<uint32_t>(hb / 2) & 1u, abort_flag, a.ws_status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t d = tbase + static_cast<uint32_t>(ab * 2 * MP + t * MP);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sw128_desc(wbuf + b * kWBytes + t * (128 * 128) + kk * 32);
              const uint64_t bd = sw128_desc(xs + h * kXHalf + kk * 32);
              mma_f16(d, ad, bd, kIdesc, !(first && h == 0 && kk == 0));
            }
          }
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
  } else if (warp >= 8) {
    // ---------------- dequantization: thread r owns row r of the block ----------------
    const int r = threadIdx.x - 256;
    const uint32_t wb0 = smem_u32(wbuf);
    const uint32_t st0 = smem_u32(stages);
    const uint32_t sw_st = static_cast<uint32_t>(r & 7) << 4;          // 128-byte swizzle of w_hat row r
    const uint32_t sw_ld = static_cast<uint32_t>((r >> 1) & 3);          // 64-byte swizzle of code row r
    uint32_t d_next = 0, z_next = 0;
    auto load_dz = [&](int u, uint32_t& dv, uint32_t& zv) {
      const int rb = u / a.Kg, g = u - rb * a.Kg;
      const int n = rb * kRows + r;
      dv = 0;
      zv = 0;
      if (n < a.N) {
        const size_t o = static_cast<size_t>(n) * a.Kg + g;
        dv = ld_nc_u16(a.scales + o);
        zv = ld_nc_u16(a.zeros + o);
      }
    };
    load_dz(u0, d_next, z_next);
    int hb = 0;
    for (int i = 0; i < cnt; ++i) {
      const int s = i % S;
      const uint32_t dv = d_next, zv = z_next;
      if (i + 1 < cnt) load_dz(u0 + i + 1, d_next, z_next);
      if (!wait_or_abort(&full[s], static_cast<uint32_t>(i / S) & 1u, abort_flag, a.ws_status)) break;
      const __half2 dd = as_h2(dv | (dv << 16));
      // 1024 + z as an fp16 pair (z is a small non-negative integer held in fp16)
      const __half zh = __hadd(__ushort_as_half(static_cast<unsigned short>(zv)), __float2half_rn(1024.0f));
      const __half2 zz = __halves2half2(zh, zh);
      const uint32_t row = st0 + s * kStageBytes + r * 64;
      uint4 c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) c[q] = lds128(row + ((static_cast<uint32_t>(q) ^ sw_ld) << 4));
      bool ok = true;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = hb & 1;
        if (hb >= 2 && !wait_or_abort(&wempty[b], static_cast<uint32_t>(hb / 2 - 1) & 1u, abort_flag, a.ws_status)) {
          ok = false;
          break;
        }
        const uint32_t dst = wb0 + b * kWBytes + r * 128;
        const uint32_t wv[8] = {c[2 * h].x,     c[2 * h].y,     c[2 * h].z,     c[2 * h].w,
                                c[2 * h + 1].x, c[2 * h + 1].y, c[2 * h + 1].z, c[2 * h + 1].w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t w = wv[j];
          sts128(dst + ((static_cast<uint32_t>(j) << 4) ^ sw_st), dq_pair(w, zz, dd), dq_pair(w >> 4, zz, dd),
                 dq_pair(w >> 8, zz, dd), dq_pair(w >> 12, zz, dd));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&wfull[b]);
        ++hb;
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[s]);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: accumulators -> y or workspace ----------------
    const int q = warp - 4;  // TMEM lane quarter
    const int te = threadIdx.x - 128;
    int f = 0, start = 0;
    for (int i = 0; i < cnt; ++i) {
      const int u = u0 + i, rb = u / a.Kg, g = u - rb * a.Kg;
      if (i == 0 || g == 0) start = i;
      if (!(i == cnt - 1 || g == a.Kg - 1)) continue;
      const int ab = f & 1;
      const bool ok = wait_or_abort(&afull[ab], static_cast<uint32_t>(f / 2) & 1u, abort_flag, a.ws_status);
      if (epi_bar_or(!ok || *abort_flag)) break;
      tc_fence_after();
      const int contrib = i - start + 1;
      const bool owner = contrib == a.Kg;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int n = rb * kRows + t * 128 + q * 32 + lane;
#pragma unroll
        for (int c = 0; c < MP / 16; ++c) {
          float v[16];
          tmem_ld16(tbase + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(ab * 2 * MP + t * MP + c * 16),
                    v);
          if (n < a.N) {
            if (owner) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (c * 16 + j < a.M) a.y[static_cast<size_t>(c * 16 + j) * a.N + n] = __float2half_rn(v[j]);
            } else {
              float4* dst = reinterpret_cast<float4*>(a.ws_acc + static_cast<size_t>(n) * MP + c * 16);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                atomicAdd(dst + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[ab]);
      ++f;
      if (!owner) {
        __threadfence();
        epi_bar();
        if (te == 0)
          *last_flag = (atomicAdd(a.ws_cnt + rb, static_cast<uint32_t>(contrib)) + contrib ==
                        static_cast<uint32_t>(a.Kg));
        epi_bar();
        if (*last_flag) {
          __threadfence();
          for (int rr = te; rr < kRows; rr += 128) {
            const int n = rb * kRows + rr;
            if (n >= a.N) continue;
            float4* src = reinterpret_cast<float4*>(a.ws_acc + static_cast<size_t>(n) * MP);
#pragma unroll
            for (int c4 = 0; c4 < MP / 4; ++c4) {
              const float4 v = __ldcg(src + c4);
              const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int j = 0; j < 4; ++j)
                if (c4 * 4 + j < a.M) a.y[static_cast<size_t>(c4 * 4 + j) * a.N + n] = __float2half_rn(vv[j]);
              src[c4] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
          if (te == 0) a.ws_cnt[rb] = 0;
        }
        epi_bar();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kCols);
  }
}

int stages_for(int mp) {
  const int stage = kCodeBytes + 2 * mp * 128;
  int s = (kMaxSmem - 1024 - 2 * kWBytes - kCtrlBytes) / stage;
  return s > kMaxStages ? kMaxStages : s;
}

template <int MP>
cudaError_t launch_mp(const TcArgs& a0, const CUtensorMap& tq, const CUtensorMap& tx, int grid, cudaStream_t st) {
  TcArgs a = a0;
  a.stages = stages_for(MP);
  if (a.stages < 2) return cudaErrorNotSupported;
  const int smem = 1024 + 2 * kWBytes + a.stages * (kCodeBytes + 2 * MP * 128) + kCtrlBytes;
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<MP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<MP><<<grid, kThreads, smem, st>>>(a, tq, tx);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmProblem& p, const Workspace& ws, cudaStream_t st) {
  if (p.M < 1 || p.M > kMaxM) return cudaErrorNotSupported;
  const int mp = (p.M + 15) / 16 * 16;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const int Kw = p.K / 8;

  // codes: u32 [N][K/8], boxes of 256 rows x 16 words (one group), 64-byte swizzle
  CUtensorMap tq, tx;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Kw), static_cast<cuuint64_t>(p.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Kw) * 4};
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
  a.scales = p.scales;
  a.zeros = p.zeros;
  a.y = p.y;
  a.ws_acc = ws.acc;
  a.ws_cnt = ws.counters;
  a.ws_status = ws.status;
  a.M = p.M;
  a.N = p.N;
  a.Kg = p.K / kGroup;
  const int row_blocks = (p.N + kRows - 1) / kRows;
  a.total_units = row_blocks * a.Kg;
  a.stages = 0;
  const int grid = min(device_sm_count(), a.total_units);
  switch (mp) {
    case 16: return launch_mp<16>(a, tq, tx, grid, st);
    case 32: return launch_mp<32>(a, tq, tx, grid, st);
    case 48: return launch_mp<48>(a, tq, tx, grid, st);
    default: return launch_mp<64>(a, tq, tx, grid, st);
  }
}

}  // namespace w4a16
