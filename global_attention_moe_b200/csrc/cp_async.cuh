// cp_async.cuh -- wrappers for the per-thread asynchronous copies (cp.async)
// the KV-cache kernel gathers K/V rows with (a row per index, so no tensor
// map applies), and for signalling their completion on an mbarrier.
#pragma once

#include "sm100.cuh"

namespace mimo {

// 16-byte asynchronous copy global -> shared; src_bytes < 16 fills the rest with
// zeros (0: nothing is read from src, which must still be a valid address).
__device__ __forceinline__ void cp_async_16(uint32_t dst_smem, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst_smem), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Arrives on `bar` once every cp.async this thread has issued so far has landed
// (without raising the barrier's pending count: the barrier expects one such
// arrival per issuing thread and phase).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Waits until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace mimo
