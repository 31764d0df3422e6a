// prefill_tc.cuh -- bf16 Lightning Attention prefill on the sm_100a tensor
// cores (tcgen05 MMAs accumulating in TMEM, operands staged by TMA).
//
// The method (section 1 of "MiniMax-01技術報告解讀以及與DeepSeek-V3對比",
// m.futurefh.com): split causal linear attention into an intra-block part
// computed with the left product and an inter-block part computed with the
// right product from a running d x d state, which avoids a cumulative sum over
// tokens.  For a 128-token block i of one sequence:
//
//     O_i  = Q_i S_{i-1}^bf16 + tril(Q_i K_i^T)^bf16 V_i      (fp32 accumulate)
//     S_i  = S_{i-1} + K_i^T V_i                               (fp32, in TMEM)
//
// Four 128x128x128 MMAs per block: MMA1 S=QK^T, MMA3 O=Q S̄, MMA4 S+=K^T V,
// MMA2 O+=P V with the masked scores P taken from TMEM.  The intra-block
// scores and the state never leave the SM; Q, K, V are read once and O is
// written once (the I/O-aware point of the first page).
//
// Sequences are cut into chunks processed in parallel (work items).  The
// state a chunk starts from is formed by a three-pass schedule: chunk_state
// (K_c^T V_c per chunk), a scan over the chunks of each sequence (exclusive
// prefixes, final state), then the main kernel started from each prefix.
// Work items come from the dense layout ([BH][N][d], chunks of equal length)
// or from packed sequences ([H][T][d] split by cu_seqlens, section 4 of the
// same page: data packing), where a chunk never crosses a sequence end.
//
// Roles in the main kernel (one CTA of 320 threads per SM, persistent):
//   warp 0     TMA producer (lane 0 issues; the warp zeroes packed tails)
//   warp 1     TMEM allocator and MMA issuer (one thread)
//   warps 2-9  two epilogue warpgroups: TMEM -> registers -> mask / convert /
//              store, warpgroup h handling columns [64h, 64h+64) of every row
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace la {
namespace tc {

// ---------------------------------------------------------------- geometry
constexpr int kStages = 2;
constexpr int kStageBytes = 3 * kTileBytes;            // Q, K, V tiles: 96 KiB
constexpr int kSbarOff = kStages * kStageBytes;        // bf16 state copy S̄ (32 KiB)
constexpr int kCtrlOff = kSbarOff + kTileBytes;        // barriers etc.
constexpr int kSmemBytes = kCtrlOff + 256 + 1024;      // + slack for 1 KiB alignment

// TMEM columns (fp32 cells; 128 lanes each)
constexpr uint32_t kColState = 0;    // S      [k-dim lanes][v-dim cols]
constexpr uint32_t kColS = 128;      // scores Q K^T
constexpr uint32_t kColP = 256;      // masked scores, bf16 pairs (64 cols)
constexpr uint32_t kColO = 384;      // output accumulator
constexpr uint32_t kTmemCols = 512;

constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);

constexpr int kModeDense = 0;
constexpr int kModeVarlen = 1;

struct Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tail_ld;      // TMA completion of a packed-sequence tail block
    uint64_t s_full;       // MMA1 complete (scores in TMEM)
    uint64_t p_ready;      // epilogue wrote P (one arrival per epilogue warp)
    uint64_t sbar_ready;   // epilogue wrote S̄ / the initial state
    uint64_t state_done;   // MMA4 complete (state updated)
    uint64_t o_full;       // MMA2 complete (output accumulated)
    uint64_t o_free;       // epilogue drained O
    uint32_t tmem_base;
    int abort;
};

// Work description shared by every kernel of the schedule.
struct Params {
    int mode;                   // kModeDense or kModeVarlen
    int Z;                      // slices of the 3-D tensor map: B*H (dense) or H (packed)
    int rows;                   // rows per slice: N (dense) or T (packed)
    int chunk_tokens;           // chunk length, a multiple of 128
    int n_chunks;               // dense: chunks per sequence
    int n_items;                // dense: Z * n_chunks (packed: read on the device)
    const int32_t* cu_seqlens;  // packed: [num_seqs + 1]
    const int32_t* chunk_off;   // packed: [num_seqs + 1] first chunk of each sequence
    const int* seq_ok;          // packed: verdict of the cu_seqlens check
    int num_seqs;
    __nv_bfloat16* o;           // [Z][rows][128]
    const float* prefix;        // [Z][chunks][128][128] exclusive chunk prefixes, or null
    float* state_out;           // [Z][128][128] written at the end of each item, or null
    float* chunk_delta;         // chunk_state output, same layout as prefix
};

struct Item {
    int z, c, t0, t1, ws;
};

__device__ __forceinline__ int num_items(const Params& p) {
    if (p.mode == kModeDense) return p.n_items;
    if (*p.seq_ok == 0) return 0;
    return p.Z * p.chunk_off[p.num_seqs];
}

__device__ __forceinline__ Item get_item(const Params& p, int item) {
    Item it;
    it.z = item % p.Z;
    const int g = item / p.Z;                     // chunk-major order
    if (p.mode == kModeDense) {
        it.c = g;
        it.t0 = g * p.chunk_tokens;
        it.t1 = min(it.t0 + p.chunk_tokens, p.rows);
        it.ws = it.z * p.n_chunks + g;
    } else {
        // sequence j with chunk_off[j] <= g < chunk_off[j+1] (empty sequences
        // own no chunk and are skipped by taking the largest such j)
        int lo = 0, hi = p.num_seqs;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.chunk_off[mid] <= g) lo = mid; else hi = mid;
        }
        it.c = g - p.chunk_off[lo];
        it.t0 = p.cu_seqlens[lo] + it.c * p.chunk_tokens;
        it.t1 = min(it.t0 + p.chunk_tokens, (int)p.cu_seqlens[lo + 1]);
        it.ws = it.z * p.chunk_off[p.num_seqs] + g;
    }
    return it;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Write 32 consecutive fp32 values of row `row` (columns col0..col0+31, col0 a
// multiple of 32) as bf16 into a [128 rows][128 cols] tile stored as two
// 128B-swizzled halves of 64 columns (the operand layout the MMAs read).
__device__ __forceinline__ void store_row32_bf16_sw128(uint8_t* tile, int row, int col0,
                                                       const uint32_t* f) {
    uint8_t* half = tile + (col0 >> 6) * kHalfBytes;
    const int chunk0 = (col0 & 63) >> 3;  // 16-byte chunks of 8 bf16
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 w;
        w.x = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 0]), __uint_as_float(f[8 * c + 1]));
        w.y = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 2]), __uint_as_float(f[8 * c + 3]));
        w.z = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 4]), __uint_as_float(f[8 * c + 5]));
        w.w = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 6]), __uint_as_float(f[8 * c + 7]));
        *reinterpret_cast<uint4*>(half + ptx::sw128_offset(row, chunk0 + c)) = w;
    }
}

// Zero rows [valid, 128) of a V tile (both 64-column halves), by one warp.
// Used for the last block of a packed sequence, whose trailing rows belong to
// the next sequence: they must not enter K^T V.
__device__ __forceinline__ void zero_tail_rows(uint8_t* vtile, int valid, int lane) {
    const int n = (kTileRows - valid) * 16;       // 16-byte chunks to clear
    for (int i = lane; i < n; i += 32) {
        const int row = valid + (i >> 4);
        const int ch = i & 15;
        *reinterpret_cast<uint4*>(vtile + (ch >> 3) * kHalfBytes + row * 128 + (ch & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// Warp-wide producer step: wait until stage `s` may be refilled, then load Q
// (optional), K and V tiles of rows [t, t+128) of slice z.  For a packed tail
// (fewer than 128 valid rows) the load completes on `tail_ld`, the warp clears
// the foreign rows of V and then releases `full`.  Returns false on abort.
template <bool kLoadQ>
__device__ __forceinline__ bool produce_tile(const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                             const CUtensorMap* tmV, uint8_t* stage_ptr,
                                             uint32_t stage, uint32_t full_bar, uint32_t tail_bar,
                                             uint32_t& n_tail, int t, int z, int valid,
                                             bool packed, uint64_t pol, int lane,
                                             volatile int* abort_flag) {
    constexpr uint32_t kBytes = (kLoadQ ? 3 : 2) * kTileBytes;
    const bool tail = packed && valid < kTileRows;
    if (lane == 0) {
        const uint32_t b = tail ? tail_bar : full_bar;
        ptx::mbar_arrive_expect_tx(b, kBytes);
        uint32_t dst = stage;
        if (kLoadQ) {
            ptx::tma_load_3d(dst, tmQ, b, 0, t, z, pol);
            ptx::tma_load_3d(dst + kHalfBytes, tmQ, b, 64, t, z, pol);
            dst += kTileBytes;
        }
        ptx::tma_load_3d(dst, tmK, b, 0, t, z, pol);
        ptx::tma_load_3d(dst + kHalfBytes, tmK, b, 64, t, z, pol);
        ptx::tma_load_3d(dst + kTileBytes, tmV, b, 0, t, z, pol);
        ptx::tma_load_3d(dst + kTileBytes + kHalfBytes, tmV, b, 64, t, z, pol);
    }
    if (!tail) return true;
    int ok = 1;
    if (lane == 0) ok = ptx::mbar_wait(tail_bar, n_tail & 1, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    ++n_tail;
    if (!ok) return false;
    zero_tail_rows(stage_ptr + (kLoadQ ? 2 : 1) * kTileBytes, valid, lane);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(full_bar);
    return true;
}

// ============================================================================
// Main kernel: outputs of every chunk from its starting state.
// ============================================================================
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kCtrlOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t sSbar = sbase + kSbarOff;
    auto bar = [&](uint64_t& b) { return ptx::smem_u32(&b); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(ctrl->full[s]), 1);
            ptx::mbar_init(bar(ctrl->empty[s]), 1);
        }
        ptx::mbar_init(bar(ctrl->tail_ld), 1);
        ptx::mbar_init(bar(ctrl->s_full), 1);
        ptx::mbar_init(bar(ctrl->p_ready), kEpiWarps);
        ptx::mbar_init(bar(ctrl->sbar_ready), kEpiWarps);
        ptx::mbar_init(bar(ctrl->state_done), 1);
        ptx::mbar_init(bar(ctrl->o_full), 1);
        ptx::mbar_init(bar(ctrl->o_free), kEpiWarps);
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&ctrl->tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmQ);
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile int* abort_flag = &ctrl->abort;
    const int n_items = num_items(p);
    const bool packed = p.mode == kModeVarlen;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = ptx::policy_evict_first();
        uint32_t g = 0, n_tail = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const Item it = get_item(p, item);
            for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                const int s = g & 1;
                if (g >= 2) {
                    int w = 1;
                    if (lane == 0) w = ptx::mbar_wait(bar(ctrl->empty[s]), ((g >> 1) + 1) & 1, abort_flag);
                    if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                }
                if (!produce_tile<true>(&tmQ, &tmK, &tmV, smem + s * kStageBytes, sbase + s * kStageBytes,
                                        bar(ctrl->full[s]), bar(ctrl->tail_ld), n_tail, t, it.z,
                                        it.t1 - t, packed, pol, lane, abort_flag)) {
                    ok = false;
                    break;
                }
            }
        }
        // Wait for the last stage releases so that no asynchronous arrive
        // is still pending on this CTA's shared memory when it exits.
        if (lane == 0)
            for (uint32_t j = (g >= 2 ? g - 2 : 0); ok && j < g; ++j)
                ok = ptx::mbar_wait(bar(ctrl->empty[j & 1]), (j >> 1) & 1, abort_flag);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = ptx::idesc_bf16(128, 128, false, false);  // Q K^T
            constexpr uint32_t id_qs = ptx::idesc_bf16(128, 128, false, true);   // Q S̄
            constexpr uint32_t id_kv = ptx::idesc_bf16(128, 128, true, true);    // K^T V
            constexpr uint32_t id_pv = ptx::idesc_bf16(128, 128, false, true);   // P V
            uint32_t g = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
                const Item it = get_item(p, item);
                bool has_state = (p.prefix != nullptr) && it.c > 0;
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    const int s = g & 1;
                    if (!ptx::mbar_wait(bar(ctrl->full[s]), (g >> 1) & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sq = sbase + s * kStageBytes;
                    const uint32_t sk = sq + kTileBytes;
                    const uint32_t sv = sq + 2 * kTileBytes;
                    // MMA1: scores = Q K^T (both operands K-major, K = head dim)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                        ptx::mma_ss(tmem + kColS, ptx::sdesc_sw128(sq + off, 16, 1024),
                                    ptx::sdesc_sw128(sk + off, 16, 1024), id_qk, kk > 0);
                    }
                    ptx::mma_commit(bar(ctrl->s_full));
                    if (!ptx::mbar_wait(bar(ctrl->sbar_ready), g & 1, abort_flag)) { ok = false; break; }
                    if (g > 0 && !ptx::mbar_wait(bar(ctrl->o_free), (g - 1) & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // MMA3: O = Q S̄ (inter-block, right product); S̄ is MN-major
                    if (has_state) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                            ptx::mma_ss(tmem + kColO, ptx::sdesc_sw128(sq + off, 16, 1024),
                                        ptx::sdesc_sw128(sSbar + kk * 2048, kHalfBytes, 1024), id_qs,
                                        kk > 0);
                        }
                    }
                    // MMA4: S += K^T V (K = tokens; both operands MN-major)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        ptx::mma_ss(tmem + kColState, ptx::sdesc_sw128(sk + kk * 2048, kHalfBytes, 1024),
                                    ptx::sdesc_sw128(sv + kk * 2048, kHalfBytes, 1024), id_kv,
                                    (kk > 0 || has_state) ? 1u : 0u);
                    }
                    ptx::mma_commit(bar(ctrl->state_done));
                    if (!ptx::mbar_wait(bar(ctrl->p_ready), g & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    // MMA2: O += P V (intra-block, left product); P from TMEM
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        ptx::mma_ts(tmem + kColO, tmem + kColP + kk * 8,
                                    ptx::sdesc_sw128(sv + kk * 2048, kHalfBytes, 1024), id_pv,
                                    (kk > 0 || has_state) ? 1u : 0u);
                    }
                    ptx::mma_commit(bar(ctrl->o_full));
                    ptx::mma_commit(bar(ctrl->empty[s]));
                    has_state = true;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;             // 0..7
        const int h = ew >> 2;               // column half owned by this warpgroup
        const int sp = warp & 3;             // TMEM sub-partition this warp may access
        const int r = sp * 32 + lane;        // tile row owned by this thread
        const int c0 = 64 * h;               // first owned column
        const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
        uint8_t* sbar_tile = smem + kSbarOff;
        uint32_t g = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const Item it = get_item(p, item);
            // ---- initial state of the chunk: TMEM S and its bf16 copy S̄
            if (p.prefix != nullptr && it.c > 0) {
                const float4* src = reinterpret_cast<const float4*>(
                    p.prefix + (size_t)it.ws * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim + c0);
                uint32_t f[64];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 x = __ldg(src + j);
                    f[4 * j + 0] = __float_as_uint(x.x);
                    f[4 * j + 1] = __float_as_uint(x.y);
                    f[4 * j + 2] = __float_as_uint(x.z);
                    f[4 * j + 3] = __float_as_uint(x.w);
                }
                ptx::tmem_st32(tl + kColState + c0, *reinterpret_cast<uint32_t(*)[32]>(f));
                ptx::tmem_st32(tl + kColState + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(f + 32));
                store_row32_bf16_sw128(sbar_tile, r, c0, f);
                store_row32_bf16_sw128(sbar_tile, r, c0 + 32, f + 32);
                ptx::tmem_st_wait();
                ptx::fence_proxy_async_smem();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->sbar_ready));

            for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                const bool last_block = t + kTileRows >= it.t1;
                // ---- 1. P = tril(scores) as bf16 pairs into TMEM (columns c0..c0+63)
                if (!ptx::mbar_wait(bar(ctrl->s_full), g & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                {
                    uint32_t pk[32];
                    if (c0 > sp * 32 + 31) {
                        // every key of this half lies above the diagonal for these rows
#pragma unroll
                        for (int j = 0; j < 32; ++j) pk[j] = 0u;
                    } else {
                        uint32_t v[64];
                        ptx::tmem_ld32(tl + kColS + c0, *reinterpret_cast<uint32_t(*)[32]>(v));
                        ptx::tmem_ld32(tl + kColS + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int key = c0 + 2 * j;
                            const float a = (key <= r) ? __uint_as_float(v[2 * j]) : 0.0f;
                            const float b = (key + 1 <= r) ? __uint_as_float(v[2 * j + 1]) : 0.0f;
                            pk[j] = ptx::pack_bf16x2(a, b);
                        }
                    }
                    ptx::tmem_st32(tl + kColP + (c0 >> 1), pk);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(ctrl->p_ready));

                // ---- 2. state: bf16 copy for the next block, or the final state
                if (!ptx::mbar_wait(bar(ctrl->state_done), g & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (!last_block || p.state_out != nullptr) {
                    uint32_t v[64];
                    ptx::tmem_ld32(tl + kColState + c0, *reinterpret_cast<uint32_t(*)[32]>(v));
                    ptx::tmem_ld32(tl + kColState + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                    ptx::tmem_ld_wait();
                    if (!last_block) {
                        store_row32_bf16_sw128(sbar_tile, r, c0, v);
                        store_row32_bf16_sw128(sbar_tile, r, c0 + 32, v + 32);
                        ptx::fence_proxy_async_smem();
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(bar(ctrl->sbar_ready));
                    } else {
                        float4* dst = reinterpret_cast<float4*>(
                            p.state_out + (size_t)it.z * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim + c0);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    }
                }

                // ---- 3. O -> bf16 -> global (columns c0..c0+63 of row t + r)
                if (!ptx::mbar_wait(bar(ctrl->o_full), g & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                {
                    uint32_t v[64];
                    ptx::tmem_ld32(tl + kColO + c0, *reinterpret_cast<uint32_t(*)[32]>(v));
                    ptx::tmem_ld32(tl + kColO + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                    ptx::tmem_ld_wait();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(ctrl->o_free));
                    if (t + r < it.t1) {
                        uint4* orow = reinterpret_cast<uint4*>(
                            p.o + ((size_t)it.z * p.rows + t + r) * kHeadDim + c0);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            uint4 w;
                            w.x = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
                            w.y = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
                            w.z = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
                            w.w = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
                            orow[j] = w;
                        }
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ============================================================================
// Pass 1: per-chunk state increment  ΔS_c = K_c^T V_c.
// ============================================================================
namespace cs {
constexpr int kStages = 3;
constexpr int kStageBytes = 2 * kTileBytes;          // K, V: 64 KiB
constexpr int kCtrlOff = kStages * kStageBytes;
constexpr int kSmemBytes = kCtrlOff + 256 + 1024;
constexpr uint32_t kTmemCols = 256;                  // two 128-column accumulators
constexpr int kThreads = 192;

struct Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tail_ld;
    uint64_t acc_full[2];
    uint64_t acc_free[2];
    uint32_t tmem_base;
    int abort;
};
}  // namespace cs

__global__ void __launch_bounds__(cs::kThreads, 1)
chunk_state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    cs::Ctrl* ctrl = reinterpret_cast<cs::Ctrl*>(smem + cs::kCtrlOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = ptx::smem_u32(smem);
    auto bar = [&](uint64_t& b) { return ptx::smem_u32(&b); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < cs::kStages; ++s) {
            ptx::mbar_init(bar(ctrl->full[s]), 1);
            ptx::mbar_init(bar(ctrl->empty[s]), 1);
        }
        ptx::mbar_init(bar(ctrl->tail_ld), 1);
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(bar(ctrl->acc_full[a]), 1);
            ptx::mbar_init(bar(ctrl->acc_free[a]), 4);
        }
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&ctrl->tmem_base), cs::kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmK);
        ptx::prefetch_tmap(&tmV);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile int* abort_flag = &ctrl->abort;
    const int n_items = num_items(p);
    const bool packed = p.mode == kModeVarlen;

    if (warp == 0) {
        // K and V are read again by the main kernel: keep them in L2 if possible.
        const uint64_t pol = ptx::policy_evict_last();
        uint32_t g = 0, n_tail = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
            const Item it = get_item(p, item);
            for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                const int s = g % cs::kStages;
                const uint32_t use = g / cs::kStages;
                if (use >= 1) {
                    int w = 1;
                    if (lane == 0) w = ptx::mbar_wait(bar(ctrl->empty[s]), (use - 1) & 1, abort_flag);
                    if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                }
                if (!produce_tile<false>(nullptr, &tmK, &tmV, smem + s * cs::kStageBytes,
                                         sbase + s * cs::kStageBytes, bar(ctrl->full[s]),
                                         bar(ctrl->tail_ld), n_tail, t, it.z, it.t1 - t, packed, pol,
                                         lane, abort_flag)) {
                    ok = false;
                    break;
                }
            }
        }
        if (lane == 0) {
            const uint32_t first = g >= (uint32_t)cs::kStages ? g - cs::kStages : 0;
            for (uint32_t j = first; ok && j < g; ++j)
                ok = ptx::mbar_wait(bar(ctrl->empty[j % cs::kStages]), (j / cs::kStages) & 1, abort_flag);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_kv = ptx::idesc_bf16(128, 128, true, true);
            uint32_t g = 0, li = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x, ++li) {
                const Item it = get_item(p, item);
                const uint32_t a = li & 1;
                if (li >= 2 && !ptx::mbar_wait(bar(ctrl->acc_free[a]), ((li >> 1) + 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                bool first = true;
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    const int s = g % cs::kStages;
                    if (!ptx::mbar_wait(bar(ctrl->full[s]), (g / cs::kStages) & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sk = sbase + s * cs::kStageBytes;
                    const uint32_t sv = sk + kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ss(tmem + a * 128, ptx::sdesc_sw128(sk + kk * 2048, kHalfBytes, 1024),
                                    ptx::sdesc_sw128(sv + kk * 2048, kHalfBytes, 1024), id_kv,
                                    (kk > 0 || !first) ? 1u : 0u);
                    ptx::mma_commit(bar(ctrl->empty[s]));
                    first = false;
                }
                if (ok) ptx::mma_commit(bar(ctrl->acc_full[a]));
            }
        }
    } else {
        const int sp = warp & 3;
        const int r = sp * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
        uint32_t li = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++li) {
            const Item it = get_item(p, item);
            const uint32_t a = li & 1;
            if (!ptx::mbar_wait(bar(ctrl->acc_full[a]), (li >> 1) & 1, abort_flag)) break;
            ptx::tc_fence_after();
            float* dst = p.chunk_delta + (size_t)it.ws * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim;
#pragma unroll
            for (int cc = 0; cc < 4; cc += 2) {
                uint32_t v[64];
                ptx::tmem_ld32(tl + a * 128 + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(v));
                ptx::tmem_ld32(tl + a * 128 + cc * 32 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                ptx::tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    reinterpret_cast<float4*>(dst + cc * 32)[j] =
                        make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                    __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->acc_free[a]));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, cs::kTmemCols);
    }
}

// ============================================================================
// Scans over chunks: exclusive prefix in place, inclusive total -> state_out.
// ============================================================================
__global__ void __launch_bounds__(256)
chunk_scan_kernel(float* ws, float* state_out, int n_chunks) {
    const int bh = blockIdx.y;
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;   // < 128*128
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float4* base = reinterpret_cast<float4*>(ws + (size_t)bh * n_chunks * (kHeadDim * kHeadDim) + e);
    constexpr int kStride4 = kHeadDim * kHeadDim / 4;
    for (int c = 0; c < n_chunks; ++c) {
        const float4 x = base[(size_t)c * kStride4];
        base[(size_t)c * kStride4] = acc;
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
    }
    if (state_out != nullptr)
        *reinterpret_cast<float4*>(state_out + (size_t)bh * (kHeadDim * kHeadDim) + e) = acc;
}

// Packed sequences: one CTA per (sequence, head) over that sequence's chunks.
// state_out is [num_seqs][H][128][128]; an empty sequence gets a zero state.
__global__ void __launch_bounds__(256)
chunk_scan_varlen_kernel(float* ws, float* state_out, const int32_t* chunk_off, const int* seq_ok,
                         int H, int num_seqs) {
    if (*seq_ok == 0) return;
    const int j = blockIdx.x;
    const int hh = blockIdx.y;
    const int total = chunk_off[num_seqs];
    const int c0 = chunk_off[j], c1 = chunk_off[j + 1];
    constexpr int kStride4 = kHeadDim * kHeadDim / 4;
    float4* base = reinterpret_cast<float4*>(ws + (size_t)hh * total * (kHeadDim * kHeadDim));
    for (int e4 = threadIdx.x; e4 < kStride4; e4 += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = c0; c < c1; ++c) {
            const float4 x = base[(size_t)c * kStride4 + e4];
            base[(size_t)c * kStride4 + e4] = acc;
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        if (state_out != nullptr)
            reinterpret_cast<float4*>(state_out + ((size_t)j * H + hh) * (kHeadDim * kHeadDim))[e4] = acc;
    }
}

// cu_seqlens check and chunk offsets of packed sequences (one CTA): verdict in
// *ok, chunk_off[j] = sum over earlier sequences of ceil(len / chunk_tokens),
// chunk_off[num_seqs] = chunks per head.  A malformed array records
// LA_ERR_BAD_SEQLENS and yields zero chunks.
__global__ void varlen_prepare_kernel(const int32_t* cu, int num_seqs, int total, int chunk_tokens,
                                      int* ok, int32_t* chunk_off) {
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int j = threadIdx.x; j <= num_seqs; j += blockDim.x) {
        const int a = cu[j];
        if ((j == 0 && a != 0) || (j == num_seqs && a != total) || a < 0 || a > total ||
            (j < num_seqs && cu[j + 1] < a))
            bad = 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        if (!bad) {
            for (int j = 0; j < num_seqs; ++j) {
                chunk_off[j] = acc;
                acc += (cu[j + 1] - cu[j] + chunk_tokens - 1) / chunk_tokens;
            }
        } else {
            for (int j = 0; j < num_seqs; ++j) chunk_off[j] = 0;
            record_device_error(LA_ERR_BAD_SEQLENS);
        }
        chunk_off[num_seqs] = acc;
        *ok = bad ? 0 : 1;
    }
}

}  // namespace tc
}  // namespace la
