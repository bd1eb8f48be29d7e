// common.cuh -- device status word and shared constants of the attention kernels.
#pragma once
#include <stdint.h>

namespace attn {

// Bits of the device status word (read and cleared by attn_get_device_status).
enum : unsigned int {
    kStatusTimeout = 1u,      // a bounded pipeline wait gave up (the CTA bailed out)
    kStatusBadPage = 2u,      // a block-table entry outside [0, num_pages) was skipped
    kStatusBadSeqLen = 4u,    // a seq_len outside [1, max_blocks * page_size) was skipped
};

// One word per device: the only state the kernels share across launches. The library is a
// single translation unit, so this definition is the only one.
__device__ unsigned int g_attn_status = 0;

__device__ __forceinline__ void raise_status(unsigned int bits) { atomicOr(&g_attn_status, bits); }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace attn
