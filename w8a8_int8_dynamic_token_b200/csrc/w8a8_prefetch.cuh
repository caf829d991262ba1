// w8a8_prefetch.cuh -- L2 prefetch of weight rows for the kernels that
// stream the weight matrix from HBM once (few activation rows).
#pragma once

#include <cstdint>

namespace w8a8 {

// Asks the memory system to bring `bytes` (a multiple of 16) of global memory
// at `src` (16-byte aligned) into L2; there is no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
               "r"(bytes)
               : "memory");
}

}  // namespace w8a8
