// async.cuh -- thin inline-PTX wrappers for sm_100a: per-thread asynchronous copies into
// shared memory (cp.async), programmatic dependent launch, and a bounded grid barrier.
#pragma once

#include <stdint.h>

namespace sfnn {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounds of waits are counted in SM clock cycles (clock64 is a cheap per-SM counter);
// 2^31 cycles is about one second at the B200's clocks.
constexpr uint64_t kWaitCycles = 1ull << 31;

// 16-byte asynchronous copy global -> shared (bypassing L1), grouped per thread.
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src_gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
// 8-byte asynchronous copy global -> shared (8-byte aligned addresses).
__device__ __forceinline__ void cp_async8(void *dst_smem, const void *src_gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
// 4-byte asynchronous copy global -> shared (4-byte aligned addresses).
__device__ __forceinline__ void cp_async4(void *dst_smem, const void *src_gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its prologue,
// and wait until the previous kernel's memory operations are visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
// nblocks.  One release-add, then acquire polls of one word; nothing is reset between
// instances or launches.  Returns false if the wait ran out after `limit` cycles (the
// caller latches an error; the counter must then be zeroed before the next launch).
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
