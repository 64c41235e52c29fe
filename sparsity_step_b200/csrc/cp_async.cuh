// Per-thread asynchronous 16-byte copies global -> shared (cp.async), used by the
// streaming kernels that keep a private ring of loads in flight per thread.
#pragma once

#include <cstdint>

namespace bl {

// 16-byte async copy global -> shared; `valid` false writes zeros (src not read). No
// compiler memory barrier: ordering comes from the commit and wait that follow.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

}  // namespace bl
