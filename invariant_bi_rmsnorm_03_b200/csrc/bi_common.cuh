// bi_common.cuh -- definitions shared by the kernels and the C-ABI layer.
#pragma once

#include <cstddef>
#include <cstdint>

#ifndef BI_INVARIANT
#define BI_INVARIANT 1
#endif

namespace bi {

// Values of the per-device status word (the first error wins).
enum : unsigned {
    BI_DEV_OK = 0,
    BI_DEV_TIMEOUT = 4,       // maps to BI_ERR_TIMEOUT
    BI_DEV_BAD_INDEX = 6,     // maps to BI_ERR_DEVICE_INDEX
};

#ifdef __CUDACC__
__device__ __forceinline__ void record_status(unsigned *status, unsigned code)
{
    atomicCAS(status, 0u, code);
}
#endif

// Default limit of one bounded wait inside a kernel.
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

constexpr int kPage = 16;        // tokens per KV-cache page
constexpr int kSplit = 256;      // keys per attention split (fixed size)

}  // namespace bi
