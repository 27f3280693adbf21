// Device helpers shared by the kernels of the w4a16 library (sm_100a only).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "the w4a16 kernels are written for sm_100a (B200) only"
#endif

namespace w4a16 {

// Device status word codes (kept in the first word of a workspace).
constexpr uint32_t kDevOk = 0;
constexpr uint32_t kDevWaitTimeout = 1;

// Every spin-wait gives up after this long (globaltimer nanoseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete.  Returns false if it
// did not complete within kWaitLimitNs; the caller records the failure.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ---- bulk copies (TMA, non-tensor form) -------------------------------------
// An L2 policy that lets streamed weights leave L2 first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Global -> this CTA's shared memory, completion counted on `bar` in bytes.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_load_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 2-D tiled tensor copy global -> this CTA's shared memory (TMA), completion
// counted on `bar` in bytes.  x is the innermost coordinate (elements); x times
// the element size must be a multiple of 16 bytes.
// Brings a tensor map (a __grid_constant__ kernel parameter) into the
// descriptor cache ahead of the first tensor copy that uses it.
__device__ __forceinline__ void prefetch_tensor_map(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 3-D tiled tensor copy global -> this CTA's shared memory (TMA); x is the
// innermost coordinate, with the same alignment rule as the 2-D form.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int x, int y, int z, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's ordinary shared-memory reads of a ring stage before the
// tensor copy (async proxy) that will next overwrite the stage.  Every thread
// that read the stage runs it before the hand-off (__syncwarp or an mbarrier
// arrival) that lets the copy be issued; without it, on B200 a refilled stage
// was seen to change under reads still in flight.
__device__ __forceinline__ void release_stage_reads() { fence_proxy_async_smem(); }

// ---- fp16 nibble unpacking ---------------------------------------------------
// (w & mask) | 0x64006400: a nibble q placed in the low mantissa bits of the
// fp16 exponent-10 binade reads as 1024 + q (bits 0..3) or 1024 + 16 q (bits 4..7).
__device__ __forceinline__ uint32_t nib_to_f16x2(uint32_t w, uint32_t mask) {
  return (w & mask) | 0x64006400u;
}

__device__ __forceinline__ __half2 as_h2(uint32_t v) {
  return *reinterpret_cast<__half2*>(&v);
}

__device__ __forceinline__ uint32_t as_u32(__half2 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

// acc + a * b with a, b fp16 and acc fp32: one rounding, to fp32 (the product is exact).
__device__ __forceinline__ float fma_f16_f32(__half a, __half b, float acc) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(__half_as_ushort(a)), "h"(__half_as_ushort(b)), "f"(acc));
  return d;
}

// Accumulates the two products of a half2 pair into two fp32 accumulators.
__device__ __forceinline__ void fma2_f16_f32(uint32_t a, uint32_t b, float& acc_lo, float& acc_hi) {
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %1, ah, bh, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(a), "r"(b));
}


// ---- packed fp32 pairs (sm_100: one instruction for two fp32 lanes) ----------
__device__ __forceinline__ uint64_t f2_pack(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return f2_pack(__float_as_uint(lo), __float_as_uint(hi));
}

__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}


__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// ---- programmatic dependent launch ---------------------------------------------
// Lets the next kernel on the stream begin launching (it still waits for this
// grid's completion in griddep_wait before using its results).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Blocks until the previous grid on the stream has completed and its memory
// operations are visible.  A no-op when the kernel was not launched with
// programmatic stream serialization.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Magic-number unpack into fp32: (w & m) | 0x4B000000 reads as 2^23 + (w & m)
// for any mask m below bit 23, so a nibble at bit 4t becomes 2^23 + 2^(4t) q.
constexpr uint32_t kMagic23 = 0x4B000000u;

}  // namespace w4a16
