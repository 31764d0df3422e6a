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
//
// Batched decode (section 3 of the same page: multi-level padding): row b of a
// batch may address a pool of states through slots[b]; a negative slot marks
// a padding row, which writes a zero output and touches no state, so a batch
// padded up to a fixed size does no state traffic for its padding.
//
// 8-bit state (the yuliangy.com digest's 8-bit quantisation): row i of a
// head's state is int8 codes c_ij and one fp32 scale a_i, S_ij = c_ij a_i.  A
// step dequantises, adds k^T v, reads o from the fp32 result and quantises each
// row again: a = m / 127, c = nearest-even of s * (127 / m), m = max_j |s_ij|,
// rows with m < 2^-100 stored as zero.  Every one of these is a single
// correctly rounded fp32 operation (no contraction), so the codes are
// reproducible bit for bit.  Traffic per head-step is 2 (d^2 + 4d) bytes
// instead of 8 d^2.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

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

// State head of batch row `head` (= b * H + h): slots[b] * H + h, or the row
// itself without a slot array.  Returns -1 for a padding row (negative slot)
// and for an out-of-range slot, which also records LA_ERR_BAD_SLOT.
__device__ __forceinline__ long long state_head(size_t head, const int32_t* slots, int H,
                                                int num_slots) {
    if (slots == nullptr) return (long long)head;
    const int b = (int)(head / (size_t)H);
    const int slot = __ldg(slots + b);
    if (slot < 0) return -1;
    if (slot >= num_slots) {
        if (threadIdx.x == 0) record_device_error(LA_ERR_BAD_SLOT);
        return -1;
    }
    return (long long)slot * H + (long long)(head % (size_t)H);
}

template <typename T, int D>
__device__ __forceinline__ void write_zero_row(T* o, size_t head) {
    if (threadIdx.x < D) o[head * D + threadIdx.x] = from_f32<T>(0.f);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   float* __restrict__ state, T* __restrict__ o, const int32_t* __restrict__ slots,
                   int H, int num_slots) {
    constexpr int kCols4 = D / 4;                    // float4 groups per row
    constexpr int kRowGroups = kThreads / kCols4;    // 8 (D=128) or 16 (D=64)
    constexpr int kRowsPer = D / kRowGroups;         // 16 (D=128) or 4 (D=64)
    static_assert(kCols4 * kRowGroups == kThreads, "layout");

    __shared__ float4 red[kRowGroups][kCols4];
    const size_t head = blockIdx.x;
    const long long sh = state_head(head, slots, H, num_slots);
    if (sh < 0) {
        write_zero_row<T, D>(o, head);
        return;
    }
    const int cg = threadIdx.x % kCols4;
    const int rg = threadIdx.x / kCols4;
    const int row0 = rg * kRowsPer;

    const T* qh = q + head * D;
    const T* kh = k + head * D;
    const T* vh = v + head * D;
    float4* S = reinterpret_cast<float4*>(state + (size_t)sh * D * D);

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


// Largest |x| over the kLanes lanes that hold one state row (a full warp at
// d = 128, a half warp at d = 64).
template <int kLanes>
__device__ __forceinline__ float row_max(float m) {
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    return m;
}

constexpr float kQ8MinRowMax = 0x1p-100f;   // rows below this are stored as zero

// Quantises the 4 values a lane holds of one row, given the row's max m;
// returns the packed codes and writes the row scale to *a.
__device__ __forceinline__ int quantize4(float4 s, float m, float* a) {
    if (m < kQ8MinRowMax) {
        *a = 0.f;
        return 0;
    }
    const float inv = __fdiv_rn(127.f, m);
    *a = __fdiv_rn(m, 127.f);
    const float xs[4] = {s.x, s.y, s.z, s.w};
    int packed = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        int c = __float2int_rn(__fmul_rn(xs[e], inv));
        c = max(-127, min(127, c));
        packed |= (c & 0xff) << (8 * e);
    }
    return packed;
}

__device__ __forceinline__ float4 dequantize4(int packed, float a) {
    float4 r;
    r.x = __fmul_rn((float)(signed char)(packed & 0xff), a);
    r.y = __fmul_rn((float)(signed char)((packed >> 8) & 0xff), a);
    r.z = __fmul_rn((float)(signed char)((packed >> 16) & 0xff), a);
    r.w = __fmul_rn((float)(signed char)((packed >> 24) & 0xff), a);
    return r;
}

// Codes of 4 values of a row given inv = fl(127 / m), m the row's max |s|.
// |s| <= m gives |y| = |fl(s * inv)| <= 127 (1 + 2^-24)^2 < 127.5, so the
// nearest integer is already within [-127, 127] and no clamp is needed; inv =
// 0 (a zero row) gives codes 0.  Rounding without a conversion instruction:
// for |y| < 2^22, t = fl(y + 1.5 * 2^23) lies in [2^23, 2^24), where the fp32
// spacing is 1, so round-to-nearest-even of the addition is exactly
// round-half-even of y, and the low byte of t's bit pattern is that integer
// modulo 256 (1.5 * 2^23 = 0x4B400000 has a zero low byte): the int8 code.
// Both operations are written _rn so that they are never contracted.
__device__ __forceinline__ int pack4_q8(float4 s, float inv) {
    constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
    const unsigned t0 = __float_as_uint(__fadd_rn(__fmul_rn(s.x, inv), kRound));
    const unsigned t1 = __float_as_uint(__fadd_rn(__fmul_rn(s.y, inv), kRound));
    const unsigned t2 = __float_as_uint(__fadd_rn(__fmul_rn(s.z, inv), kRound));
    const unsigned t3 = __float_as_uint(__fadd_rn(__fmul_rn(s.w, inv), kRound));
    const unsigned lo = __byte_perm(t0, t1, 0x0040u);   // t0.b0, t1.b0
    const unsigned hi = __byte_perm(t2, t3, 0x0040u);   // t2.b0, t3.b0
    return (int)__byte_perm(lo, hi, 0x5410u);
}

// The 4 int8 codes of a word as exact fp32 values, without a conversion
// instruction: flipping the sign bit of a byte b gives b + 128 in [0, 255];
// placed in the low mantissa byte under exponent 0x4B it reads 2^23 + b + 128,
// and subtracting 2^23 + 128 leaves b exactly.
__device__ __forceinline__ float4 codes_to_f32(int packed) {
    constexpr float kBias = 8388736.0f;     // 2^23 + 128
    const unsigned u = (unsigned)packed ^ 0x80808080u;
    float4 r;
    r.x = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u)), kBias);
    r.y = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7441u)), kBias);
    r.z = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7442u)), kBias);
    r.w = __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7443u)), kBias);
    return r;
}

// Packed (two fp32 lanes per instruction, sm_100) forms of the same steps.
// Each half is the identical correctly rounded fp32 operation as the scalar
// form.  The packed multiply may be fused by the compiler with a packed add
// that consumes it (one rounding instead of two: near-tie codes moved by one
// when that happened), so no packed product here feeds a packed add: the
// quantising product stays a scalar __fmul_rn, which is never contracted, and
// the dequantising product feeds only the addend of a fused multiply-add.
struct Row4 {
    float2 lo, hi;   // columns 4c, 4c+1 and 4c+2, 4c+3
};

__device__ __forceinline__ Row4 codes_to_f32x2(int packed) {
    constexpr float kBias = 8388736.0f;     // 2^23 + 128, as in codes_to_f32
    const unsigned u = (unsigned)packed ^ 0x80808080u;
    const float2 nb = make_float2(-kBias, -kBias);
    Row4 r;
    r.lo = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u)),
                                  __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7441u))), nb);
    r.hi = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7442u)),
                                  __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7443u))), nb);
    return r;
}

__device__ __forceinline__ int pack4_q8x2(const Row4& s, float inv) {
    constexpr float kRound = 12582912.0f;   // 1.5 * 2^23, as in pack4_q8
    const float2 rr = make_float2(kRound, kRound);
    const float2 tl = __fadd2_rn(make_float2(__fmul_rn(s.lo.x, inv), __fmul_rn(s.lo.y, inv)), rr);
    const float2 th = __fadd2_rn(make_float2(__fmul_rn(s.hi.x, inv), __fmul_rn(s.hi.y, inv)), rr);
    const unsigned lo = __byte_perm(__float_as_uint(tl.x), __float_as_uint(tl.y), 0x0040u);
    const unsigned hi = __byte_perm(__float_as_uint(th.x), __float_as_uint(th.y), 0x0040u);
    return (int)__byte_perm(lo, hi, 0x5410u);
}

// N consecutive values of a row-vector (q or k rows of one lane) as fp32,
// with 16- or 8-byte loads (the offsets used are multiples of the load size).
template <typename T, int N>
__device__ __forceinline__ void load_f32(const T* p, float (&out)[N]);
template <>
__device__ __forceinline__ void load_f32<float, 16>(const float* p, float (&out)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(p) + i);
        out[4 * i] = t.x;
        out[4 * i + 1] = t.y;
        out[4 * i + 2] = t.z;
        out[4 * i + 3] = t.w;
    }
}
template <>
__device__ __forceinline__ void load_f32<float, 4>(const float* p, float (&out)[4]) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = t.x;
    out[1] = t.y;
    out[2] = t.z;
    out[3] = t.w;
}
__device__ __forceinline__ void unpack_bf16x2(unsigned w, float& lo, float& hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
}
template <>
__device__ __forceinline__ void load_f32<__nv_bfloat16, 16>(const __nv_bfloat16* p, float (&out)[16]) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 t = __ldg(reinterpret_cast<const uint4*>(p) + i);
        unpack_bf16x2(t.x, out[8 * i + 0], out[8 * i + 1]);
        unpack_bf16x2(t.y, out[8 * i + 2], out[8 * i + 3]);
        unpack_bf16x2(t.z, out[8 * i + 4], out[8 * i + 5]);
        unpack_bf16x2(t.w, out[8 * i + 6], out[8 * i + 7]);
    }
}
template <>
__device__ __forceinline__ void load_f32<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&out)[4]) {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
    unpack_bf16x2(t.x, out[0], out[1]);
    unpack_bf16x2(t.y, out[2], out[3]);
}

// Maxima of R rows whose values are spread over L lanes each (R <= L, powers
// of two), as a butterfly that halves the rows it carries at every exchange:
// after log2(R) exchanges lane l of a row's L lanes holds a partial max of
// row l / (L / R), which the remaining log2(L / R) exchanges complete.  That
// is R - 1 + log2(L / R) shuffles instead of R log2(L), and afterwards each
// row's max sits in L / R lanes, so the row's divisions run once per warp
// instruction for R rows at a time.
template <int R, int L>
__device__ __forceinline__ float row_max_scatter(const float (&lm)[R], int lane_in_row) {
    float cur[R];
#pragma unroll
    for (int r = 0; r < R; ++r) cur[r] = lm[r];
#pragma unroll
    for (int n = R, off = L / 2; n > 1; n >>= 1, off >>= 1) {
        const bool upper = (lane_in_row & off) != 0;
#pragma unroll
        for (int r = 0; r < n / 2; ++r) {
            const float send = upper ? cur[r] : cur[r + n / 2];
            const float keep = upper ? cur[r + n / 2] : cur[r];
            cur[r] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
        }
    }
#pragma unroll
    for (int off = L / (2 * R); off > 0; off >>= 1)
        cur[0] = fmaxf(cur[0], __shfl_xor_sync(0xffffffffu, cur[0], off));
    return cur[0];
}

// One decode step on the 8-bit state.  Persistent CTAs walk the batch rows
// (b, h) with a stride of the grid; thread 0 streams each row's codes and
// scales into a ring of kQ8Stages shared-memory stages with bulk copies
// (cp.async.bulk, completion on an mbarrier), so the loads of the next rows
// overlap the arithmetic of this one.  Compute layout as decode_step_kernel:
// a lane owns 4 value columns (one 32-bit word of codes) of kRowsPer rows, and
// the kCols4 lanes of a row are consecutive lanes of one warp.  The rows'
// maxima come from row_max_scatter; the lanes holding a row's max compute its
// 127 / m and m / 127 and pass 127 / m back by shuffle.  New codes and scales
// go straight from registers to global memory.
constexpr int kQ8Stages = 4;

template <int D>
struct Q8Smem {
    static constexpr int kCodeBytes = D * D;
    static constexpr int kScaleBytes = D * 4;
    static constexpr int kStageBytes = kCodeBytes + kScaleBytes;
    static constexpr int kRowGroups = kThreads / (D / 4);
    static constexpr int kRedOff = kQ8Stages * kStageBytes;                 // float4 red[2][groups][D/4]
    static constexpr int kCtrlOff = kRedOff + 2 * kRowGroups * (D / 4) * 16;
    static constexpr int kBytes = kCtrlOff + 128;                           // mbarriers, slot ids, flag
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2)
decode_step_q8_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      int8_t* __restrict__ codes, float* __restrict__ scales, T* __restrict__ o,
                      const int32_t* __restrict__ slots, int H, int num_slots, long long n_rows) {
    using L = Q8Smem<D>;
    constexpr int kCols4 = D / 4;                       // lanes per row
    constexpr int kRowGroups = L::kRowGroups;
    constexpr int kRowsPer = D / kRowGroups;            // rows per lane
    constexpr int kHolders = kCols4 / kRowsPer;         // lanes holding one row's max
    static_assert(kCols4 * kRowGroups == kThreads && kRowsPer % 4 == 0 && kRowsPer <= kCols4, "layout");

    extern __shared__ __align__(128) uint8_t smem[];
    float4* red = reinterpret_cast<float4*>(smem + L::kRedOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kCtrlOff);
    long long* stage_head = reinterpret_cast<long long*>(smem + L::kCtrlOff + 8 * kQ8Stages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kCtrlOff + 16 * kQ8Stages);
    auto bar = [&](int s) { return ptx::smem_u32(bars + s); };
    const uint32_t stage0 = ptx::smem_u32(smem);

    const long long G = gridDim.x;
    // thread 0: resolve the slot of the j-th row of this CTA and start its copies
    auto issue = [&](long long j) {
        const long long r = blockIdx.x + j * G;
        if (r >= n_rows) return;
        const int s = (int)(j % kQ8Stages);
        const long long sh = state_head((size_t)r, slots, H, num_slots);
        stage_head[s] = sh;
        if (sh < 0) {
            ptx::mbar_arrive(bar(s));
            return;
        }
        ptx::mbar_arrive_expect_tx(bar(s), L::kStageBytes);
        const uint32_t dst = stage0 + s * L::kStageBytes;
        ptx::bulk_load(dst, codes + (size_t)sh * L::kCodeBytes, L::kCodeBytes, bar(s));
        ptx::bulk_load(dst + L::kCodeBytes, scales + (size_t)sh * D, L::kScaleBytes, bar(s));
    };
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kQ8Stages; ++s) ptx::mbar_init(bar(s), 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        for (int j = 0; j < kQ8Stages; ++j) issue(j);

    const int cg = threadIdx.x % kCols4;
    const int rg = threadIdx.x / kCols4;
    const int row0 = rg * kRowsPer;
    long long j = 0;
    for (; blockIdx.x + j * G < n_rows; ++j) {
        const size_t head = (size_t)(blockIdx.x + j * G);
        const int s = (int)(j % kQ8Stages);
        float kr[kRowsPer], qr[kRowsPer], vc[4];
        load_f32<T, kRowsPer>(k + head * D + row0, kr);
        load_f32<T, kRowsPer>(q + head * D + row0, qr);
        load_f32<T, 4>(v + head * D + 4 * cg, vc);
        const bool ok = ptx::mbar_wait(bar(s), (uint32_t)((j / kQ8Stages) & 1), abort_flag);
        const long long sh = stage_head[s];
        float4* red_j = red + (j & 1) * (kRowGroups * kCols4);
        if (ok && sh >= 0) {
            const uint8_t* st = smem + s * L::kStageBytes;
            const int* Cs = reinterpret_cast<const int*>(st);
            const float* As = reinterpret_cast<const float*>(st + L::kCodeBytes);
            Row4 x[kRowsPer];
            float lm[kRowsPer];
            float2 acc_lo = make_float2(0.f, 0.f), acc_hi = make_float2(0.f, 0.f);
            const float2 v_lo = make_float2(vc[0], vc[1]), v_hi = make_float2(vc[2], vc[3]);
#pragma unroll
            for (int i = 0; i < kRowsPer; ++i) {
                const float2 ai = make_float2(As[row0 + i], As[row0 + i]);
                const float2 ki = make_float2(kr[i], kr[i]);
                const float2 qi = make_float2(qr[i], qr[i]);
                x[i] = codes_to_f32x2(Cs[(row0 + i) * kCols4 + cg]);
                // s = fma(k_i, v_j, c_ij * a_i), then o += q_i s
                x[i].lo = __ffma2_rn(ki, v_lo, __fmul2_rn(x[i].lo, ai));
                x[i].hi = __ffma2_rn(ki, v_hi, __fmul2_rn(x[i].hi, ai));
                acc_lo = __ffma2_rn(qi, x[i].lo, acc_lo);
                acc_hi = __ffma2_rn(qi, x[i].hi, acc_hi);
                lm[i] = fmaxf(fmaxf(fabsf(x[i].lo.x), fabsf(x[i].lo.y)), fmaxf(fabsf(x[i].hi.x), fabsf(x[i].hi.y)));
            }
            const float m = row_max_scatter<kRowsPer, kCols4>(lm, cg);
            const bool zero_row = m < kQ8MinRowMax;
            const float inv_mine = zero_row ? 0.f : __fdiv_rn(127.f, m);
            const float a_mine = zero_row ? 0.f : __fdiv_rn(m, 127.f);
            int* C = reinterpret_cast<int*>(codes + (size_t)sh * L::kCodeBytes);
            if (cg % kHolders == 0) scales[(size_t)sh * D + row0 + cg / kHolders] = a_mine;
#pragma unroll
            for (int i = 0; i < kRowsPer; ++i) {
                const float inv = __shfl_sync(0xffffffffu, inv_mine, i * kHolders, kCols4);
                __stcs(C + (size_t)(row0 + i) * kCols4 + cg, pack4_q8x2(x[i], inv));
            }
            const float4 acc = make_float4(acc_lo.x, acc_lo.y, acc_hi.x, acc_hi.y);
            red_j[rg * kCols4 + cg] = acc;
        }
        // every thread is done with stage s and has written its partial sums
        if (__syncthreads_or(!ok)) break;
        if (threadIdx.x == 0) issue(j + kQ8Stages);
        if (sh < 0) {
            write_zero_row<T, D>(o, head);
        } else if (rg == 0) {
            float4 t = red_j[cg];
#pragma unroll
            for (int g = 1; g < kRowGroups; ++g) {
                const float4 u = red_j[g * kCols4 + cg];
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
    // after a timeout: let the copies already issued land (bounded) before exit
    if (threadIdx.x == 0 && *abort_flag) {
        for (long long jj = j; jj < j + kQ8Stages && blockIdx.x + jj * G < n_rows; ++jj) {
            const unsigned long long t0 = globaltimer_ns();
            while (!ptx::mbar_try_wait(bar((int)(jj % kQ8Stages)), (uint32_t)((jj / kQ8Stages) & 1)) &&
                   globaltimer_ns() - t0 < wait_limit_ns()) {
            }
        }
    }
}

// fp32 states -> 8-bit form.  A warp takes 32 / (D/4) rows at a time (D/4
// lanes per row), grid-stride over warps; all lanes of a warp run the same
// iterations, so the row-max shuffles always have the full warp.
template <int D>
__global__ void __launch_bounds__(256)
state_quantize_q8_kernel(const float* __restrict__ S, int8_t* __restrict__ codes,
                         float* __restrict__ scales, long long rows) {
    constexpr int kLanes = D / 4;
    constexpr int kRowsPerWarp = 32 / kLanes;
    const int lane = threadIdx.x & 31;
    const int cg = lane % kLanes;
    const long long warps = (long long)gridDim.x * (blockDim.x / 32);
    const long long warp = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    for (long long r0 = warp * kRowsPerWarp; r0 < rows; r0 += warps * kRowsPerWarp) {
        const long long r = r0 + lane / kLanes;
        const bool live = r < rows;
        const float4 x = live ? __ldcs(reinterpret_cast<const float4*>(S + r * D) + cg)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        const float m = row_max<kLanes>(fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
        float a;
        const int packed = quantize4(x, m, &a);
        if (live) {
            reinterpret_cast<int*>(codes + r * D)[cg] = packed;
            if (cg == 0) scales[r] = a;
        }
    }
}

// 8-bit form -> fp32 states, S_ij = c_ij * a_i; one float4 per thread, grid-stride.
template <int D>
__global__ void __launch_bounds__(256)
state_dequantize_q8_kernel(const int8_t* __restrict__ codes, const float* __restrict__ scales,
                           float* __restrict__ S, long long n4) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const int packed = reinterpret_cast<const int*>(codes)[i];
        reinterpret_cast<float4*>(S)[i] = dequantize4(packed, scales[i / (D / 4)]);
    }
}

}  // namespace decode
}  // namespace la
