// Shared-to-global bulk copies (cp.async.bulk), used by the kernels that
// assemble whole output rows in shared memory: the block-mask builder and the
// q-side transpose.
#pragma once
#include <cstdint>

namespace bsmt {

// Copies `bytes` (a multiple of 16) from shared to global memory with the
// bulk copy engine; both addresses 16-byte aligned. Completion is tracked by
// the thread's bulk async-groups (bulk_commit_group / bulk_wait_group*).
__device__ __forceinline__ void bulk_store_1d(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

}  // namespace bsmt
