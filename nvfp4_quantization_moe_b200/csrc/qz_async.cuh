// qz_async.cuh -- asynchronous global -> shared copies for the staged kernels (sm_100a).
#pragma once

#include <stdint.h>

namespace qz {

// ---------------------------------------------------------------------------
// asynchronous global -> shared copies (cp.async, 16 bytes, zero-filled past
// src_bytes); each thread waits for its own groups, a CTA barrier publishes
// them to the other threads
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace qz
