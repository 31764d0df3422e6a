// tokens.cuh -- token-order reversal of [Z][N][row] tensors, for the
// anti-causal sums of the backward pass (sum over t >= s is the causal sum of
// the reversed sequence).
#pragma once

#include "common.cuh"

namespace la {

// dst[z][N-1-t] = src[z][t]; rows of row16 16-byte words; src != dst.
__global__ void __launch_bounds__(256)
reverse_tokens_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long Z, long N, int row16) {
    const long total = Z * N * row16;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const long c = i % row16;
        const long t = (i / row16) % N;
        const long z = i / (row16 * N);
        dst[(z * N + (N - 1 - t)) * row16 + c] = __ldcs(src + i);
    }
}

}  // namespace la
