// async.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, 1-D bulk async copies
// (the TMA engine's cp.async.bulk, no multicast), programmatic dependent launch, and a
// grid-wide barrier.  Every wait here is bounded: after `limit` polls it reports failure
// instead of spinning forever.
#pragma once

#include <stdint.h>

namespace sfnn {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the same condition.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounds of waits are counted in SM clock cycles (clock64 is a cheap per-SM counter);
// 2^31 cycles is about one second at the B200's clocks.
constexpr uint64_t kWaitCycles = 1ull << 31;

// Wait for the phase with the given parity to complete; false after `limit` cycles.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit) {
  const uint64_t t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((uint64_t)(clock64() - t0) > limit) return false;
  }
}

// global -> shared bulk copy completing on an mbarrier (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its prologue,
// and wait until the previous kernel's memory operations are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t atom_add_release_gpu_u64(uint64_t *p, uint64_t v) {
  uint64_t old;
  asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

// Grid barrier over `nblocks` co-resident CTAs, called by ONE thread per CTA, on a 64-bit
// arrival counter that only grows: the ticket an arrival draws names its barrier instance
// (ticket / nblocks), which completes when the counter reaches the next multiple of
// nblocks.  One release-add and acquire polls; nothing is reset between instances or
// launches.  Returns false if the wait ran out after `limit` cycles (the caller latches
// an error; the counter must then be zeroed before the next launch).
__device__ __forceinline__ bool grid_barrier(uint64_t *count, uint32_t nblocks, uint64_t limit) {
  const uint64_t ticket = atom_add_release_gpu_u64(count, 1ull);
  const uint64_t target = (ticket / nblocks + 1) * nblocks;
  const uint64_t t0 = clock64();
  for (;;) {
    if (ld_acquire_gpu_u64(count) >= target) return true;
    if ((uint64_t)(clock64() - t0) > limit) return false;
  }
}

}  // namespace sfnn
