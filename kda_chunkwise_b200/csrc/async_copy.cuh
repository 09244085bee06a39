// Small asynchronous global->shared copies used next to cp_async_16 (mma_frag.cuh).
#pragma once

#include <cstdint>

namespace kda {

// 4-byte asynchronous global->shared copy (completes with cp.async.wait_group / wait_all)
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}

}  // namespace kda
