// decode.cuh -- one decode step of causal linear attention for every (b, h):
//
//     S <- S + k^T v ;   o = q S
//
// (section 3 of "MiniMax-01技術報告解讀以及與DeepSeek-V3對比": prefill and
// decode are executed separately; the recurrence is the fixed-size state of
// the closing analogy of "MiniMax M2.1").  The step is bound by HBM traffic:
// the fp32 state (d*d*4 bytes per head) is read and written once, against
// 4*d*d flops.  One CTA of 256 threads per head; each thread owns a float4
// column group of D/ROW_GROUPS rows, so every warp-wide access is a run of
// 512 contiguous bytes; the per-column partial sums of o are combined across
// row groups through shared memory.
#pragma once

#include "common.cuh"

namespace la {
namespace decode {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr int kThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   float* __restrict__ state, T* __restrict__ o) {
    constexpr int kCols4 = D / 4;                    // float4 groups per row
    constexpr int kRowGroups = kThreads / kCols4;    // 8 (D=128) or 16 (D=64)
    constexpr int kRowsPer = D / kRowGroups;         // 16 (D=128) or 4 (D=64)
    static_assert(kCols4 * kRowGroups == kThreads, "layout");

    __shared__ float4 red[kRowGroups][kCols4];
    const size_t head = blockIdx.x;
    const int cg = threadIdx.x % kCols4;
    const int rg = threadIdx.x / kCols4;
    const int row0 = rg * kRowsPer;

    const T* qh = q + head * D;
    const T* kh = k + head * D;
    const T* vh = v + head * D;
    float4* S = reinterpret_cast<float4*>(state + head * D * D);

    // Issue all state loads first (memory-level parallelism), then the update.
    float4 s[kRowsPer];
#pragma unroll
    for (int i = 0; i < kRowsPer; ++i) s[i] = __ldcs(S + (size_t)(row0 + i) * kCols4 + cg);

    const float v0 = to_f32(vh[4 * cg + 0]), v1 = to_f32(vh[4 * cg + 1]);
    const float v2 = to_f32(vh[4 * cg + 2]), v3 = to_f32(vh[4 * cg + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kRowsPer; ++i) {
        const float ki = to_f32(kh[row0 + i]);
        const float qi = to_f32(qh[row0 + i]);
        float4 x = s[i];
        x.x = fmaf(ki, v0, x.x);
        x.y = fmaf(ki, v1, x.y);
        x.z = fmaf(ki, v2, x.z);
        x.w = fmaf(ki, v3, x.w);
        __stcs(S + (size_t)(row0 + i) * kCols4 + cg, x);
        acc.x = fmaf(qi, x.x, acc.x);
        acc.y = fmaf(qi, x.y, acc.y);
        acc.z = fmaf(qi, x.z, acc.z);
        acc.w = fmaf(qi, x.w, acc.w);
    }
    red[rg][cg] = acc;
    __syncthreads();
    if (rg == 0) {
        float4 t = red[0][cg];
#pragma unroll
        for (int g = 1; g < kRowGroups; ++g) {
            const float4 u = red[g][cg];
            t.x += u.x;
            t.y += u.y;
            t.z += u.z;
            t.w += u.w;
        }
        T* oh = o + head * D;
        oh[4 * cg + 0] = from_f32<T>(t.x);
        oh[4 * cg + 1] = from_f32<T>(t.y);
        oh[4 * cg + 2] = from_f32<T>(t.z);
        oh[4 * cg + 3] = from_f32<T>(t.w);
    }
}

}  // namespace decode
}  // namespace la
