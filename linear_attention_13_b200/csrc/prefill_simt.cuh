// prefill_simt.cuh -- fp32 Lightning Attention prefill on the CUDA cores.
//
// Same block algorithm as the tensor-core path (section 1 of
// "MiniMax-01技術報告解讀以及與DeepSeek-V3對比": intra-block left product,
// inter-block right product from the running state), in plain fp32 FMA with
// no TF32 rounding, for fp32 inputs.  For block i of `blk` tokens:
//
//     O_i = Q_i S_{i-1} + tril(Q_i K_i^T) V_i ,   S_i = S_{i-1} + K_i^T V_i
//
// One CTA per sequence segment (a (b, h) row range of the dense layout, or a
// (head, packed sequence) of the varlen layout).  The d x d state stays in
// shared memory; a block is processed in sub-tiles of 32 query rows and 32 key
// rows so that any blk >= 1 fits.
#pragma once

#include "common.cuh"

namespace la {
namespace simt {

constexpr int kThreads = 256;
constexpr int kSub = 32;

template <int D>
constexpr int smem_bytes() {
    // S[D][D] + Qs[32][D] + Ks[32][D] + Vs[32][D] + scores[32][33]
    return (D * D + 3 * kSub * D + kSub * (kSub + 1)) * 4;
}

// Segment description: element offset of token 0 of the segment's head in
// q/k/v/o, its token range, and where its final state goes.
struct Segment {
    size_t base;       // element offset of token row 0 of this head
    int t0, t1;        // token range [t0, t1)
    float* state;      // [D][D] destination or null
    const float* state_in;  // [D][D] starting state, or null (zero)
};

template <int D>
__device__ void run_segment(const float* __restrict__ q, const float* __restrict__ k,
                            const float* __restrict__ v, float* __restrict__ o, const Segment sg,
                            int blk, float* smem) {
    float* S = smem;                     // [D][D]
    float* Qs = S + D * D;               // [32][D]
    float* Ks = Qs + kSub * D;           // [32][D]
    float* Vs = Ks + kSub * D;           // [32][D]
    float* P = Vs + kSub * D;            // [32][33]
    const int tid = threadIdx.x;

    for (int i = tid; i < D * D; i += kThreads) S[i] = sg.state_in ? sg.state_in[i] : 0.f;
    __syncthreads();

    // thread -> (row i, columns j = jc + 8*m) of a 32 x D output sub-tile
    constexpr int kColsPer = D / 8;
    const int oi = tid >> 3;
    const int jc = tid & 7;

    for (int b0 = sg.t0; b0 < sg.t1; b0 += blk) {
        const int b1 = min(b0 + blk, sg.t1);
        for (int qs = b0; qs < b1; qs += kSub) {
            const int qe = min(qs + kSub, b1);
            for (int x = tid; x < kSub * D; x += kThreads) {
                const int rr = x / D, cc = x % D;
                Qs[x] = (qs + rr < qe) ? q[sg.base + (size_t)(qs + rr) * D + cc] : 0.f;
            }
            __syncthreads();
            // inter-block: Q S_{i-1}
            float acc[kColsPer];
#pragma unroll
            for (int m = 0; m < kColsPer; ++m) {
                const int j = jc + 8 * m;
                float a = 0.f;
                for (int c = 0; c < D; ++c) a = fmaf(Qs[oi * D + c], S[c * D + j], a);
                acc[m] = a;
            }
            // intra-block: tril(Q K^T) V over key sub-tiles up to the diagonal
            for (int ks = b0; ks < qe; ks += kSub) {
                const int ke = min(ks + kSub, qe);
                for (int x = tid; x < kSub * D; x += kThreads) {
                    const int rr = x / D, cc = x % D;
                    const bool in = ks + rr < ke;
                    Ks[x] = in ? k[sg.base + (size_t)(ks + rr) * D + cc] : 0.f;
                    Vs[x] = in ? v[sg.base + (size_t)(ks + rr) * D + cc] : 0.f;
                }
                __syncthreads();
                for (int x = tid; x < kSub * kSub; x += kThreads) {
                    const int rr = x / kSub, cc = x % kSub;
                    float sc = 0.f;
                    if (ks + cc <= qs + rr) {
                        for (int c = 0; c < D; ++c) sc = fmaf(Qs[rr * D + c], Ks[cc * D + c], sc);
                    }
                    P[rr * (kSub + 1) + cc] = sc;
                }
                __syncthreads();
#pragma unroll
                for (int m = 0; m < kColsPer; ++m) {
                    const int j = jc + 8 * m;
                    float a = acc[m];
                    for (int c = 0; c < kSub; ++c) a = fmaf(P[oi * (kSub + 1) + c], Vs[c * D + j], a);
                    acc[m] = a;
                }
                __syncthreads();
            }
            if (qs + oi < qe) {
#pragma unroll
                for (int m = 0; m < kColsPer; ++m) o[sg.base + (size_t)(qs + oi) * D + jc + 8 * m] = acc[m];
            }
            __syncthreads();
        }
        // S_i = S_{i-1} + K_i^T V_i
        for (int ks = b0; ks < b1; ks += kSub) {
            const int ke = min(ks + kSub, b1);
            for (int x = tid; x < kSub * D; x += kThreads) {
                const int rr = x / D, cc = x % D;
                const bool in = ks + rr < ke;
                Ks[x] = in ? k[sg.base + (size_t)(ks + rr) * D + cc] : 0.f;
                Vs[x] = in ? v[sg.base + (size_t)(ks + rr) * D + cc] : 0.f;
            }
            __syncthreads();
            for (int x = tid; x < D * D; x += kThreads) {
                const int i = x / D, j = x % D;
                float a = S[x];
                for (int c = 0; c < kSub; ++c) a = fmaf(Ks[c * D + i], Vs[c * D + j], a);
                S[x] = a;
            }
            __syncthreads();
        }
    }
    if (sg.state != nullptr)
        for (int x = tid; x < D * D; x += kThreads) sg.state[x] = S[x];
}

// Dense layout: one CTA per (b, h).
template <int D>
__global__ void __launch_bounds__(kThreads)
prefill_simt_kernel(const float* q, const float* k, const float* v, float* o, float* state_out,
                    const float* state_in, int N, int blk) {
    extern __shared__ float smem_f[];
    const int bh = blockIdx.x;
    Segment sg;
    sg.base = (size_t)bh * N * D;
    sg.t0 = 0;
    sg.t1 = N;
    sg.state = state_out ? state_out + (size_t)bh * D * D : nullptr;
    sg.state_in = state_in ? state_in + (size_t)bh * D * D : nullptr;
    run_segment<D>(q, k, v, o, sg, blk, smem_f);
}

// Varlen layout [H][T][D]: one CTA per (sequence, head); `seqlens_ok` is the
// verdict of the cu_seqlens check, nothing is touched when it is zero.
template <int D>
__global__ void __launch_bounds__(kThreads)
prefill_simt_varlen_kernel(const float* q, const float* k, const float* v, float* o,
                           float* state_out, const float* state_in, const int32_t* cu_seqlens,
                           const int* seqlens_ok, int num_seqs, int H, int T, int blk) {
    extern __shared__ float smem_f[];
    if (*seqlens_ok == 0) return;
    const int j = blockIdx.x;
    const int h = blockIdx.y;
    Segment sg;
    sg.base = (size_t)h * T * D;
    sg.t0 = cu_seqlens[j];
    sg.t1 = cu_seqlens[j + 1];
    sg.state = state_out ? state_out + ((size_t)j * H + h) * D * D : nullptr;
    sg.state_in = state_in ? state_in + ((size_t)j * H + h) * D * D : nullptr;
    run_segment<D>(q, k, v, o, sg, blk, smem_f);
}

}  // namespace simt

// cu_seqlens check: cu[0] == 0, non-decreasing, cu[num_seqs] == total.  Writes
// the verdict to *ok (1 good, 0 bad) and records LA_ERR_BAD_SEQLENS if bad.
// Single CTA; total work num_seqs + 1 reads.
__global__ void check_seqlens_kernel(const int32_t* cu, int num_seqs, int total, int* ok) {
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int j = threadIdx.x; j <= num_seqs; j += blockDim.x) {
        const int a = cu[j];
        if (j == 0 && a != 0) bad = 1;
        if (j == num_seqs && a != total) bad = 1;
        if (j < num_seqs && cu[j + 1] < a) bad = 1;
        if (a < 0 || a > total) bad = 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        *ok = bad ? 0 : 1;
        if (bad) record_device_error(LA_ERR_BAD_SEQLENS);
    }
}

}  // namespace la
