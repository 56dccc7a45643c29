// TMA tensor maps, mbarriers and bounded waits (sm_100a).
//
// Every wait on an mbarrier is bounded: after kWaitNs of polling it gives up,
// reports MOE_DEVICE_ERR_TIMEOUT and lets the caller run on to the kernel's
// end through the same barriers, so no CTA can spin forever.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

// A wait gives up after kWaitNs of global time.  A polling thread may be
// suspended up to kSuspendNs per try_wait (woken early when the phase
// completes), so waiting warps do not steal issue slots.
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kSuspendNs = 20000;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tensor core).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Waits for the phase of parity `parity` to complete; false (and a status
// bit) if it did not within kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  report(status, MOE_DEVICE_ERR_TIMEOUT);
  return false;
}

// Abort protocol of the warp-specialised kernels (TMA producer, consumers,
// and for tcgen05 an MMA issuer).  Every wait is
// bounded; a wait that runs out reports MOE_DEVICE_ERR_TIMEOUT and sets the
// CTA's abort flag, and a wait in progress elsewhere in the CTA gives up as
// soon as it sees the flag.  A role whose wait fails leaves its loop at once,
// so after an abort nothing issues another TMA copy, MMA, commit or barrier
// arrival.  Before the CTA exits, the TMA producer waits (bounded) until
// every stage it issued has landed, and the MMA issuer commits a drain
// barrier that the TMEM owner waits on, so no asynchronous copy or MMA is in
// flight when shared memory and TMEM are released.

// Bounded wait that gives up after a timeout anywhere in the CTA (abort).
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, int32_t *status, volatile int32_t *abort) {
  if (*abort) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitNs) break;
  }
  report(status, MOE_DEVICE_ERR_TIMEOUT);
  *abort = 1;
  return false;
}

// Waits (bounded, whatever the abort flag says) until the last `issued` TMA
// stages of a ring of `stages` full-barriers have landed.  Stage j of the
// issue order used barrier j % stages in phase j / stages.
__device__ __forceinline__ void tma_drain(uint64_t *full, uint32_t issued, uint32_t stages, int32_t *status) {
  const uint32_t first = issued > stages ? issued - stages : 0;
  for (uint32_t j = first; j < issued; ++j) mbar_wait(&full[j % stages], (j / stages) & 1, status);
}

// 2-D tiled TMA load (no multicast) completing on `bar`.  c0 is the inner
// coordinate; c0 * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 1-D bulk copy global -> shared completing on `bar` (16-byte aligned
// addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 16 bytes global -> shared by the issuing thread (L2 only), tracked by
// commit groups (cp_async_commit / cp_async_wait<n>).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most n of this thread's committed groups are still in flight.
template <int n>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Host: 2-D tensor map over a row-major [outer, inner] array.
bool make_map_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                 uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace moe
