// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tiled loads and
// stores, 1-D bulk copies and async-proxy fences. Every copy here reads
// and writes this CTA's own shared memory only.
#pragma once

#include <cuda.h>
#include <cstdint>

namespace srftq {

// Device guard word: bit 0 = a bounded mbarrier wait gave up; bit 1 = an
// index check of the debug build (SRFTQ_DEBUG_CHECKS) failed.
constexpr unsigned kGuardWaitTimeout = 1u;
constexpr unsigned kGuardIndex = 2u;

#ifdef SRFTQ_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Index check of the debug build: returns whether an access may go ahead.
// In the debug build a failed check records kGuardIndex in the guard word
// (the access is then skipped by the caller); nothing traps. In the release
// build it is the constant true and compiles away.
__device__ __forceinline__ bool dbg_ok(bool ok, unsigned* guard) {
  if constexpr (kDebugChecks) {
    if (!ok) atomicOr(guard, kGuardIndex);
    return ok;
  } else {
    return true;
  }
}

// try_wait polls suspend the thread for a hardware-defined slice (well under
// a microsecond each); 1 << 22 of them bound a wait to a few seconds at most.
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Plain arrival (count 1) without transaction bytes.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete; gives up after kWaitLimit
// polls and returns false (the caller records the guard and stops).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  return false;
}

// 4-D tiled TMA load global -> shared, completion counted on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_addr(bar))
      : "memory");
}

// 4-D tiled TMA store shared -> global (rows outside the tensor are clipped).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_addr(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// 1-D bulk copy global -> shared; dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N committed store groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Byte offset inside a TMA box written with the 32/64/128-byte swizzle: the
// 16-byte chunk index (address bits 4..) is XORed with the 128-byte row index
// (address bits 7..), masked to the swizzle span. SPAN == 16 means no swizzle.
template <int SPAN>
__device__ __forceinline__ uint32_t swizzle(uint32_t off) {
  if constexpr (SPAN <= 16) {
    return off;
  } else {
    constexpr uint32_t mask = SPAN / 16 - 1;
    return off ^ (((off >> 7) & mask) << 4);
  }
}

// 16-byte shared-memory load / store at a 32-bit shared address.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// 8-byte shared-memory load / store at a 32-bit shared address.
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts64(uint32_t addr, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(v.x), "r"(v.y) : "memory");
}

// Row r of a swizzled TMA box of rows of SPAN bytes: the 16-byte chunk c of
// the row sits at  base + r * SPAN + ((c ^ (r' & mask)) << 4), r' = the
// 128-byte line index of the row. For a row whose offset has no bits inside
// the chunk field, that is (base + r * SPAN + (x << 4)) ^ (c << 4) with
// x = r' & mask: swz_row() returns that per-row term, swz_chunk() applies
// the chunk XOR (base 1024-aligned, piece offsets multiples of 1024).
template <int SPAN>
__device__ __forceinline__ uint32_t swz_row(uint32_t base, uint32_t r) {
  const uint32_t off = r * SPAN;
  if constexpr (SPAN <= 16) {
    return base + off;
  } else {
    constexpr uint32_t mask = SPAN / 16 - 1;
    return base + (off | (((off >> 7) & mask) << 4));
  }
}

template <int SPAN>
__device__ __forceinline__ uint32_t swz_chunk(uint32_t row_addr, uint32_t c) {
  return SPAN <= 16 ? row_addr + 16 * c : row_addr ^ (16 * c);
}

}  // namespace srftq
