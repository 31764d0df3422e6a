// common.cuh -- shared definitions of the CUDA path (status word, sizes).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "lightning.h"

namespace la {

// Device-side status word: the first error any kernel records wins (atomicCAS
// from LA_OK).  la_get_last_error() reads and clears it.  The library is one
// translation unit, so this is its only definition.
__device__ int g_device_status = 0;

__device__ __forceinline__ void record_device_error(int code) {
    atomicCAS(&g_device_status, (int)LA_OK, code);
}

// Bounded waits give up after g_wait_limit_ns nanoseconds of %globaltimer
// (la_set_wait_limit_ns changes it; kDefaultWaitLimitNs by default).  Read
// only once a wait has not completed at its first test.
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;  // 2 s
__device__ unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;

__device__ __forceinline__ unsigned long long wait_limit_ns() { return g_wait_limit_ns; }

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Tile geometry of the tensor-core path: 128-row tiles, head dim 128, bf16
// operands split into two 64-column halves of 128-byte rows (the 128B-swizzle
// atom width).
constexpr int kTileRows = 128;
constexpr int kHeadDim = 128;
constexpr int kHalfBytes = kTileRows * 128;      // 16 KiB: 128 rows x 64 bf16
constexpr int kTileBytes = 2 * kHalfBytes;       // 32 KiB: 128 x 128 bf16

}  // namespace la
