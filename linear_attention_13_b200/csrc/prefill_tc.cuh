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
// Four kernels carry the outputs, each a persistent, warp-specialised CTA
// per SM (roles listed at each kernel): prefill_tc_kernel (whole value rows,
// single pass with look-back over chunk states, or 64-token blocks),
// prefill_seq_kernel and prefill_seq64_kernel (value columns split over two
// CTAs, one MMA issuer per product, 128- or 64-token blocks) and
// chunk_state_kernel (the first pass of the three-pass schedule).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace la {
namespace tc {

// ---------------------------------------------------------------- geometry
// Shared memory of the main kernel for a CTA handling kNV value columns: two
// stages of Q, K (128 x 128) and V (128 x kNV) tiles, the bf16 state copy S̄
// (128 x kNV), then the barriers.
constexpr int kStages = 2;
__host__ __device__ constexpr int stage_bytes(int nv) { return 2 * kTileBytes + (nv / 64) * kHalfBytes; }
__host__ __device__ constexpr int sbar_offset(int nv) { return kStages * stage_bytes(nv); }
__host__ __device__ constexpr int ctrl_offset(int nv) { return sbar_offset(nv) + (nv / 64) * kHalfBytes; }
__host__ __device__ constexpr int smem_bytes(int nv) { return ctrl_offset(nv) + 512 + 1024; }

// TMEM columns (fp32 cells; 128 lanes each)
constexpr uint32_t kColState = 0;    // S      [k-dim lanes][v-dim cols]
constexpr uint32_t kColS = 128;      // scores Q K^T; the masked scores P (bf16
                                     // pairs) overwrite columns [128,160) (keys
                                     // 0-63) and [192,224) (keys 64-127)
constexpr uint32_t kColO = 256;      // output accumulator
constexpr uint32_t kColDelta = 384;  // single pass: chunk increment K_c^T V_c
constexpr uint32_t kTmemCols = 512;

// TMEM column of the bf16 P pairs for keys [16*kk, 16*kk+16): each epilogue
// thread writes its packed keys into the first half of the score columns it
// has just read itself.
__host__ __device__ constexpr uint32_t p_col(int kk) {
    return kColS + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
}

// Same for 64-token blocks (scores 64 x 64): keys [32h, 32h+32) are packed
// into columns [32h, 32h+16) of the score area.
__host__ __device__ constexpr uint32_t p_col64(int kk) {
    return kColS + (kk < 2 ? kk * 8 : 32 + (kk - 2) * 8);
}

// 14 warps: warp 0 producer, warp 1 MMA issuer, warps 2-9 epilogue, warps
// 10-13 chain warps.
constexpr int kEpiWarps = 8;       // P / S̄ / O / final state: 64 columns of one row per thread
constexpr int kChainWarps = 4;     // phase B (single pass) and starting states, full rows
constexpr int kFirstEpiWarp = 2;
constexpr int kFirstChainWarp = kFirstEpiWarp + kEpiWarps;
constexpr int kThreads = 32 * (kFirstChainWarp + kChainWarps);

constexpr int kModeDense = 0;
constexpr int kModeVarlen = 1;

// Work items of prefill_tc_kernel pass from its producer to the other roles
// through a ring of kRing entries; each is read by the MMA issuer, the 8
// epilogue warps and the 4 chain warps.
constexpr int kRing = 4;
constexpr int kRingReaders = 1 + kEpiWarps + kChainWarps;

struct Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];     // every MMA of the tile done (V and Q no longer read)
    uint64_t k_empty[kStages];   // K no longer read (the tile's last MMA4 done)
    uint64_t tail_ld;      // TMA completion of a packed-sequence tail block
    uint64_t s_full;       // MMA1 complete (scores in TMEM)
    uint64_t p_ready;      // epilogue wrote P (one arrival per epilogue warp)
    uint64_t sbar_ready;   // epilogue released / initialised TMEM S and wrote S̄
    uint64_t state_done;   // MMA4 complete (state updated)
    uint64_t o_full;       // MMA2 complete (output accumulated)
    uint64_t o_free;       // epilogue drained O
    uint64_t delta_done;   // single pass: chunk increment K_c^T V_c complete
    uint64_t delta_free;   // single pass: chain warps read the increment
    uint64_t state_free;   // epilogue finished with TMEM S / S̄ of an item
    uint64_t o_staged;     // every epilogue warp wrote its part of O (bf16) to smem
    uint64_t o_stored[kStages];  // O tile staged in stage s has left shared memory
    uint64_t ring_full[kRing];   // ring entry written by the producer
    uint64_t ring_free[kRing];   // ring entry read by every reader (kRingReaders)
    uint64_t drain;              // the issuer's last MMAs complete (teardown)
    int ring[kRing];             // item of each claimed position (n_items: no more)
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Ctrl) <= 512, "control block");

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
    float* state_out;           // final states, or null: dense [Z][128][128], packed
                                // [num_seqs][H][128][128]
    float* chunk_delta;         // chunk_state output, same layout as prefix
    int fused;                  // single pass: chunk prefixes found by look-back
    float* chain;               // single pass: inclusive chunk prefixes, layout of prefix
    int* flags;                 // single pass: "prefix published" words, one per chunk,
                                // value part and chain warp ([chunks][vparts][4], zeroed)
    int vparts;                 // value columns split over this many CTAs (1 or 2)
    int blk;                    // block size of the intra/inter split: 128, or 64 (vparts 1)
    const int32_t* seq_order;   // packed, one chunk per sequence: the sequence of chunk g
                                // (non-empty sequences, longest first), or null
    const float* state_in;      // starting state of every sequence (layout of state_out),
                                // or null (zero)
    int* ticket;                // single pass: item counter (zeroed with the flags); a
                                // CTA takes its items from it in increasing order, so
                                // an item's predecessor chunk has always been taken by
                                // a CTA that is running.  Null: items by static stride
    int ticket_base;            // first item the counter hands out (0)
    int stall_tile;             // split kernels: 1 + the CTA tile count whose loads the
                                // producer leaves unissued (a test hook), or 0
};

// One work item: rows [t0, t1) of slice z, chunk c of its sequence, value
// columns [vp * 128 / vparts, (vp + 1) * 128 / vparts).
//   ws    index of the chunk in the per-chunk state arrays
//   sidx  index of the sequence's final state in state_out
//   last  the chunk ends its sequence
struct Item {
    int z, c, t0, t1, ws, sidx, vp;
    bool last;
};

__device__ __forceinline__ int num_items(const Params& p) {
    if (p.mode == kModeDense) return p.n_items;
    if (*p.seq_ok == 0) return 0;
    return p.Z * p.chunk_off[p.num_seqs] * p.vparts;
}

// Items are ordered chunk-major, then slice, then value part: the value parts
// of one chunk are neighbours (they run together and share Q and K in L2).
__device__ __forceinline__ Item get_item(const Params& p, int item) {
    Item it;
    it.vp = item % p.vparts;
    item /= p.vparts;
    it.z = item % p.Z;
    const int g = item / p.Z;
    if (p.mode == kModeDense) {
        it.c = g;
        it.t0 = g * p.chunk_tokens;
        it.t1 = min(it.t0 + p.chunk_tokens, p.rows);
        it.ws = it.z * p.n_chunks + g;
        it.sidx = it.z;
        it.last = g == p.n_chunks - 1;
    } else if (p.seq_order != nullptr) {
        // one chunk per sequence, longest sequences first (so that the work
        // of a persistent grid is balanced)
        const int j = p.seq_order[g];
        it.c = 0;
        it.t0 = p.cu_seqlens[j];
        it.t1 = p.cu_seqlens[j + 1];
        it.ws = it.z * p.chunk_off[p.num_seqs] + g;
        it.sidx = j * p.Z + it.z;
        it.last = true;
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
        it.sidx = lo * p.Z + it.z;
        it.last = g == p.chunk_off[lo + 1] - 1;
    }
    return it;
}

// Starting state of an item that is not found by look-back, or null (zero).
// With a prefix array (three-pass) it is the chunk's exclusive prefix, which
// the scan starts from state_in, so chunk 0 reads it there too: state_out may
// then alias state_in although the scan writes the final state before this
// pass runs.  Without one, chunk 0 starts from the caller's state_in.  Points
// at row 0, column 0 of the d x d state.
__device__ __forceinline__ const float* start_state(const Params& p, const Item& it) {
    if (it.c == 0 && p.state_in == nullptr) return nullptr;
    if (p.prefix != nullptr) return p.prefix + (size_t)it.ws * (kHeadDim * kHeadDim);
    return it.c == 0 ? p.state_in + (size_t)it.sidx * (kHeadDim * kHeadDim) : nullptr;
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

// The same for 16 values (col0 a multiple of 16).
__device__ __forceinline__ void store_row16_bf16_sw128(uint8_t* tile, int row, int col0,
                                                       const uint32_t* f) {
    uint8_t* half = tile + (col0 >> 6) * kHalfBytes;
    const int chunk0 = (col0 & 63) >> 3;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint4 w;
        w.x = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 0]), __uint_as_float(f[8 * c + 1]));
        w.y = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 2]), __uint_as_float(f[8 * c + 3]));
        w.z = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 4]), __uint_as_float(f[8 * c + 5]));
        w.w = ptx::pack_bf16x2(__uint_as_float(f[8 * c + 6]), __uint_as_float(f[8 * c + 7]));
        *reinterpret_cast<uint4*>(half + ptx::sw128_offset(row, chunk0 + c)) = w;
    }
}

// Zero rows [valid, 128) of a V tile of `halves` 64-column halves, by one
// warp.  Used for the last block of a packed sequence, whose trailing rows
// belong to the next sequence: they must not enter K^T V.
__device__ __forceinline__ void zero_tail_rows(uint8_t* vtile, int valid, int lane, int halves) {
    const int n = (kTileRows - valid) * 8 * halves;   // 16-byte chunks to clear
    for (int i = lane; i < n; i += 32) {
        const int row = valid + i / (8 * halves);
        const int ch = i % (8 * halves);
        *reinterpret_cast<uint4*>(vtile + (ch >> 3) * kHalfBytes + row * 128 + (ch & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// Tensor maps of one call.  q, k, v describe [Z][rows][128] bf16 as
// {64 columns, rows, 2 column halves, Z} with a {64, 128, 2, 1} box: one TMA
// operation moves a whole 128-row tile, both 64-column halves (128B swizzle),
// into two consecutive 16 KiB halves.  A TMA engine moves about one operation
// per 200 ns per issuing thread, so whole-tile operations double what one
// producer thread loads.  v_half and o are {128, rows, Z} maps with a
// {64, 128, 1} box: one half tile of V (split value columns) or of O.
struct TileMaps {
    CUtensorMap q, k, v, v_half, o, k_half;
};

// Warp-wide producer step: wait until stage `s` may be refilled, then load Q
// (optional), K and V tiles of rows [t, t+128) of slice z.  For a packed tail
// (fewer than 128 valid rows) the load completes on `tail_ld`, the warp clears
// the foreign rows of V and then releases `full`.  Returns false on abort.
// The V tile holds kVHalves 64-column halves starting at column v_x.  L2
// policies: q_pol for Q, pol for K, v_pol (0: pol) for V.
template <bool kLoadQ, int kVHalves = 2>
__device__ __forceinline__ bool produce_tile(const TileMaps& maps, uint8_t* stage_ptr,
                                             uint32_t stage, uint32_t full_bar, uint32_t tail_bar,
                                             uint32_t& n_tail, int t, int z, int valid,
                                             bool packed, uint64_t q_pol, uint64_t pol, int lane,
                                             volatile int* abort_flag, int v_x = 0, uint64_t v_pol = 0) {
    constexpr uint32_t kBytes = (kLoadQ ? 2 : 1) * kTileBytes + kVHalves * kHalfBytes;
    const bool tail = packed && valid < kTileRows;
    if (lane == 0) {
        const uint32_t b = tail ? tail_bar : full_bar;
        ptx::mbar_arrive_expect_tx(b, kBytes);
        uint32_t dst = stage;
        if (kLoadQ) {
            ptx::tma_load_4d(dst, &maps.q, b, 0, t, 0, z, q_pol);
            dst += kTileBytes;
        }
        ptx::tma_load_4d(dst, &maps.k, b, 0, t, 0, z, pol);
        if (kVHalves == 2)
            ptx::tma_load_4d(dst + kTileBytes, &maps.v, b, 0, t, 0, z, v_pol ? v_pol : pol);
        else
            ptx::tma_load_3d(dst + kTileBytes, &maps.v_half, b, v_x, t, z, v_pol ? v_pol : pol);
    }
    if (!tail) return true;
    int ok = 1;
    if (lane == 0) ok = ptx::mbar_wait(tail_bar, n_tail & 1, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    ++n_tail;
    if (!ok) return false;
    zero_tail_rows(stage_ptr + (kLoadQ ? 2 : 1) * kTileBytes, valid, lane, kVHalves);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(full_bar);
    return true;
}

// ============================================================================
// Main kernel: outputs of every chunk from its starting state.
//
// Three-pass schedule (p.fused == 0): the starting state of chunk c > 0 is
// the exclusive prefix p.prefix[ws] written by chunk_state + chunk_scan.
//
// Single pass (p.fused == 1), per work item (z, c):
//   phase A  a chunk with a successor accumulates its increment K_c^T V_c in
//            TMEM (columns kColDelta);
//   phase B  the epilogue waits for the inclusive prefix of chunk c-1, which
//            the CTA owning it publishes in global memory, publishes its own
//            inclusive prefix for chunk c+1, and loads the exclusive prefix
//            as the starting state;
//   phase C  outputs, as in the three-pass schedule.
// A CTA runs phase A of its next item before phase C of the current one, so
// the K/V stream of that phase A overlaps the epilogue's phase B.  Items are
// visited in chunk-major order and every CTA walks its items in increasing
// order, so the smallest unfinished item never waits (the predecessor it
// needs has a smaller index).  Every wait is bounded; a consumed prefix is
// dropped from L2 without write-back (it has exactly one reader).
// ============================================================================
// kNV: value columns handled by one CTA (128, or 64 when the columns of every
// head are split over p.vparts = 2 CTAs).  Columns of S and O are independent
// (S[:, v] = sum k^T v[v], O[:, v] = Q S[:, v] + P V[:, v]), so a split needs
// no exchange; both parts compute the scores Q K^T.
//
// kBlk: block size of the intra/inter split, 128 or 64.  With 64, each 128-row
// tile is processed as two 64-token blocks: scores Q_b K_b^T (64 x 64), Q_b S̄
// and P_b V_b run as M = 64 tcgen05 MMAs (rows in TMEM lanes 16 i .. 16 i + 15
// of each 32-lane sub-partition i), and the state is updated every 64 tokens.
template <int kNV, int kBlk = 128>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ TileMaps maps,
                  const Params p) {
    static_assert(kNV == 64 || kNV == 128, "value part width");
    static_assert(kBlk == 128 || (kBlk == 64 && kNV == 128), "block size");
    constexpr int kSub = kTileRows / kBlk;     // blocks per 128-row tile
    constexpr int kVHalves = kNV / 64;
    constexpr int kStageB = stage_bytes(kNV);
    constexpr int kSbarOffT = sbar_offset(kNV);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + ctrl_offset(kNV));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t sSbar = sbase + kSbarOffT;
    auto bar = [&](uint64_t& b) { return ptx::smem_u32(&b); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(ctrl->full[s]), 1);
            ptx::mbar_init(bar(ctrl->empty[s]), 1);
            ptx::mbar_init(bar(ctrl->k_empty[s]), 1);
        }
        ptx::mbar_init(bar(ctrl->tail_ld), 1);
        ptx::mbar_init(bar(ctrl->s_full), 1);
        ptx::mbar_init(bar(ctrl->p_ready), kEpiWarps);
        ptx::mbar_init(bar(ctrl->sbar_ready), kEpiWarps);
        ptx::mbar_init(bar(ctrl->state_done), 1);
        ptx::mbar_init(bar(ctrl->o_full), 1);
        ptx::mbar_init(bar(ctrl->o_free), kEpiWarps);
        ptx::mbar_init(bar(ctrl->delta_done), 1);
        ptx::mbar_init(bar(ctrl->delta_free), kChainWarps);
        ptx::mbar_init(bar(ctrl->state_free), kEpiWarps);
        ptx::mbar_init(bar(ctrl->o_staged), kEpiWarps);
        for (int s = 0; s < kStages; ++s) ptx::mbar_init(bar(ctrl->o_stored[s]), 1);
        for (int i = 0; i < kRing; ++i) {
            ptx::mbar_init(bar(ctrl->ring_full[i]), 1);
            ptx::mbar_init(bar(ctrl->ring_free[i]), kRingReaders);
        }
        ptx::mbar_init(bar(ctrl->drain), 1);
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&ctrl->tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&maps.q);
        ptx::prefetch_tmap(&maps.k);
        ptx::prefetch_tmap(&maps.v);
        ptx::prefetch_tmap(&maps.v_half);
        ptx::prefetch_tmap(&maps.o);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile int* abort_flag = &ctrl->abort;
    const int n_items = num_items(p);
    const bool packed = p.mode == kModeVarlen;
    const bool fused = p.fused != 0;
    const int stride = gridDim.x;
    // phase A is run for chunks that have a successor (single pass only)
    auto has_phase_a = [&](const Item& it) { return fused && !it.last; };
    // Item at ring position j (the CTA's j-th item; n_items = none), once the
    // producer has written it; false on abort.
    auto read_pos = [&](uint32_t j, int& item) -> bool {
        const uint32_t slot = j % kRing;
        if (!ptx::mbar_wait(bar(ctrl->ring_full[slot]), (j / kRing) & 1, abort_flag)) return false;
        item = *reinterpret_cast<volatile int*>(&ctrl->ring[slot]);
        return true;
    };
    auto release_pos = [&](uint32_t j) { ptx::mbar_arrive(bar(ctrl->ring_free[j % kRing])); };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_first = ptx::policy_evict_first();
        const uint64_t pol_last = ptx::policy_evict_last();
        // with split value columns the other CTA of the head reads the same Q
        // and K: keep them at normal priority, evict only the private V half early
        const uint64_t pol_qk = p.vparts > 1 ? ptx::policy_evict_normal() : pol_first;
        uint32_t g = 0, n_tail = 0;
        bool ok = true;
        uint32_t c_uses[kStages] = {0, 0};   // phase-C uses of each stage so far
        // the last load into each stage (its barrier and phase parity), which
        // the teardown after an abort lets land
        uint32_t ld_bar0 = 0, ld_par0 = 0, ld_bar1 = 0, ld_par1 = 0;
        // One tile (rows [t, t+128) of item it) into stage g & 1.  Each operand
        // is loaded as soon as its slot is free: K once the stage's previous
        // tile finished MMA4 (k_empty), V once it finished MMA2 (empty), and Q
        // (phase C) once the O tile staged in the Q slot has been stored.
        auto produce = [&](const Item& it, int t, bool phase_c) -> bool {
            const int s = g & 1;
            const uint32_t stage = sbase + s * kStageB;
            const bool tail = packed && it.t1 - t < kTileRows;
            const uint32_t fb = tail ? bar(ctrl->tail_ld) : bar(ctrl->full[s]);
            const uint64_t pol_k = phase_c ? pol_qk : pol_last;
            const uint64_t pol_v = phase_c ? pol_first : pol_last;
            int w = 1;
            if (lane == 0) {
                if (g >= 2) w = ptx::mbar_wait(bar(ctrl->k_empty[s]), ((g >> 1) + 1) & 1, abort_flag);
                if (w) {
                    // K counts on the phase now; the arrival comes with V (and Q)
                    ptx::mbar_expect_tx(fb, kTileBytes);
                    if (s == 0) { ld_bar0 = fb; ld_par0 = tail ? (n_tail & 1) : ((g >> 1) & 1); }
                    else { ld_bar1 = fb; ld_par1 = tail ? (n_tail & 1) : ((g >> 1) & 1); }
                    ptx::tma_load_4d(stage + kTileBytes, &maps.k, fb, 0, t, 0, it.z, pol_k);
                    if (g >= 2) w = ptx::mbar_wait(bar(ctrl->empty[s]), ((g >> 1) + 1) & 1, abort_flag);
                    if (w && phase_c && c_uses[s] > 0)
                        w = ptx::mbar_wait(bar(ctrl->o_stored[s]), (c_uses[s] - 1) & 1, abort_flag);
                    if (w) {
                        ptx::mbar_arrive_expect_tx(fb, (phase_c ? kTileBytes : 0) + kVHalves * kHalfBytes);
                        if (kVHalves == 2)
                            ptx::tma_load_4d(stage + 2 * kTileBytes, &maps.v, fb, 0, t, 0, it.z, pol_v);
                        else
                            ptx::tma_load_3d(stage + 2 * kTileBytes, &maps.v_half, fb, it.vp * kNV, t, it.z, pol_v);
                        if (phase_c) ptx::tma_load_4d(stage, &maps.q, fb, 0, t, 0, it.z, pol_qk);
                    } else {
                        // aborted after K: close the phase on K alone, so that the
                        // teardown can wait for it to land
                        ptx::mbar_arrive(fb);
                    }
                }
            }
            if (!__shfl_sync(0xffffffffu, w, 0)) return false;
            if (phase_c) ++c_uses[s];
            if (tail) {
                // a packed tail: clear the next sequence's rows of V, then release
                if (lane == 0) w = ptx::mbar_wait(bar(ctrl->tail_ld), n_tail & 1, abort_flag);
                ++n_tail;
                if (!__shfl_sync(0xffffffffu, w, 0)) return false;
                zero_tail_rows(smem + s * kStageB + 2 * kTileBytes, it.t1 - t, lane, kVHalves);
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(ctrl->full[s]));
            }
            return true;
        };
        auto load_phase_a = [&](const Item& it) {
            // K and V only, kept in L2 for phase C
            for (int t = it.t0; ok && t < it.t1; t += kTileRows, ++g)
                if (!produce(it, t, false)) ok = false;
        };
        // ---- work items: taken here -- from the ticket counter in the single
        //      pass (so that items start in increasing order across the grid),
        //      by a static stride otherwise -- and handed to the other roles
        //      through the ring.  Returns the item (n_items: none), -1 on abort.
        uint32_t n_claimed = 0;
        bool ended = false;
        auto claim = [&]() -> int {
            int item = n_items, w = 1;
            if (lane == 0) {
                const uint32_t slot = n_claimed % kRing;
                if (n_claimed >= (uint32_t)kRing)
                    w = ptx::mbar_wait(bar(ctrl->ring_free[slot]), ((n_claimed / kRing) + 1) & 1, abort_flag);
                if (w) {
                    if (!ended) {
                        item = p.ticket != nullptr ? p.ticket_base + atomicAdd(p.ticket, 1)
                                                   : (int)blockIdx.x + (int)n_claimed * stride;
                        item = min(item, n_items);
                    }
                    *reinterpret_cast<volatile int*>(&ctrl->ring[slot]) = item;
                    ptx::mbar_arrive(bar(ctrl->ring_full[slot]));
                }
            }
            w = __shfl_sync(0xffffffffu, w, 0);
            item = __shfl_sync(0xffffffffu, item, 0);
            if (!w) return -1;
            ended = ended || item >= n_items;
            ++n_claimed;
            return item;
        };
        int cur = claim();
        if (cur >= 0 && cur < n_items) {
            const Item first = get_item(p, cur);
            if (has_phase_a(first)) load_phase_a(first);
        }
        while (ok && cur >= 0 && cur < n_items) {
            const Item it = get_item(p, cur);
            const int nxi = claim();
            if (nxi < 0) { ok = false; break; }
            if (nxi < n_items) {
                const Item nx = get_item(p, nxi);
                if (has_phase_a(nx)) load_phase_a(nx);
            }
            for (int t = it.t0; ok && t < it.t1; t += kTileRows, ++g)
                if (!produce(it, t, true)) ok = false;
            cur = nxi;
        }
        if (cur < 0) ok = false;
        // Wait for the last stage releases (MMA commits and O stores) so that no
        // asynchronous arrive is still pending on this CTA's shared memory when
        // it exits.
        if (lane == 0) {
            for (uint32_t j = (g >= 2 ? g - 2 : 0); ok && j < g; ++j) {
                ok = ptx::mbar_wait(bar(ctrl->k_empty[j & 1]), (j >> 1) & 1, abort_flag);
                if (ok) ok = ptx::mbar_wait(bar(ctrl->empty[j & 1]), (j >> 1) & 1, abort_flag);
            }
            for (int s = 0; ok && s < kStages; ++s)
                if (c_uses[s] > 0) ok = ptx::mbar_wait(bar(ctrl->o_stored[s]), (c_uses[s] - 1) & 1, abort_flag);
            if (!ok) {
                // after an abort: let the loads already issued land (bounded)
                if (ld_bar0) ptx::mbar_drain(ld_bar0, ld_par0);
                if (ld_bar1) ptx::mbar_drain(ld_bar1, ld_par1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_qk = ptx::idesc_bf16(kBlk, kBlk, false, false);  // Q K^T
            constexpr uint32_t id_qs = ptx::idesc_bf16(kBlk, kNV, false, true);    // Q S̄
            constexpr uint32_t id_kv = ptx::idesc_bf16(128, kNV, true, true);      // K^T V
            constexpr uint32_t id_pv = ptx::idesc_bf16(kBlk, kNV, false, true);    // P V
            uint32_t g = 0, n_sb = 0, n_a = 0, n_blk = 0;
            bool ok = true, issued = false;
            // phase A: TMEM delta = K_c^T V_c over the chunk's blocks
            auto run_phase_a = [&](const Item& it) {
                if (n_a > 0 && !ptx::mbar_wait(bar(ctrl->delta_free), (n_a - 1) & 1, abort_flag)) {
                    ok = false;
                    return;
                }
                ptx::tc_fence_after();
                bool first = true;
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    const int s = g & 1;
                    if (!ptx::mbar_wait(bar(ctrl->full[s]), (g >> 1) & 1, abort_flag)) { ok = false; return; }
                    ptx::tc_fence_after();
                    const uint32_t sk = sbase + s * kStageB + kTileBytes;
                    const uint32_t sv = sk + kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ss(tmem + kColDelta, ptx::sdesc_sw128(sk + kk * 2048, kHalfBytes, 1024),
                                    ptx::sdesc_sw128(sv + kk * 2048, kHalfBytes, 1024), id_kv,
                                    (kk > 0 || !first) ? 1u : 0u);
                    ptx::mma_commit(bar(ctrl->k_empty[s]));
                    ptx::mma_commit(bar(ctrl->empty[s]));
                    first = false;
                    issued = true;
                }
                ptx::mma_commit(bar(ctrl->delta_done));
                ++n_a;
            };
            uint32_t pos = 0;
            int cur = n_items;
            if (!read_pos(0, cur)) ok = false;
            if (ok && cur < n_items) {
                const Item first = get_item(p, cur);
                if (has_phase_a(first)) run_phase_a(first);
            }
            for (; ok && cur < n_items; ++pos) {
                const Item it = get_item(p, cur);
                int nxi = n_items;
                if (!read_pos(pos + 1, nxi)) { ok = false; break; }
                if (nxi < n_items) {
                    const Item nx = get_item(p, nxi);
                    if (has_phase_a(nx)) run_phase_a(nx);
                    if (!ok) break;
                }
                bool has_state = fused ? (it.c > 0 || p.state_in != nullptr) : start_state(p, it) != nullptr;
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    const int s = g & 1;
                    if (!ptx::mbar_wait(bar(ctrl->full[s]), (g >> 1) & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sq = sbase + s * kStageB;
                    const uint32_t sk = sq + kTileBytes;
                    const uint32_t sv = sq + 2 * kTileBytes;
                    const int nsub = (kSub == 1 || it.t1 - t > kBlk) ? kSub : 1;
                    for (int sb = 0; sb < nsub; ++sb, ++n_blk) {
                        // rows [sb * kBlk, (sb + 1) * kBlk) of the tile: kBlk rows of
                        // 128 bytes into each 64-column half
                        const uint32_t roff = (uint32_t)sb * kBlk * 128;
                        // MMA1: scores = Q K^T (both operands K-major, K = head dim).
                        // It overwrites the P of the previous block, whose MMA2 was
                        // issued earlier by this thread (tcgen05 MMAs run in order).
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32 + roff;
                            ptx::mma_ss(tmem + kColS, ptx::sdesc_sw128(sq + off, 16, 1024),
                                        ptx::sdesc_sw128(sk + off, 16, 1024), id_qk, kk > 0);
                        }
                        ptx::mma_commit(bar(ctrl->s_full));
                        if (!ptx::mbar_wait(bar(ctrl->sbar_ready), n_sb++ & 1, abort_flag)) { ok = false; break; }
                        if (n_blk > 0 && !ptx::mbar_wait(bar(ctrl->o_free), (n_blk - 1) & 1, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
                        // MMA3: O = Q S̄ (inter-block, right product); S̄ is MN-major
                        if (has_state) {
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32 + roff;
                                ptx::mma_ss(tmem + kColO, ptx::sdesc_sw128(sq + off, 16, 1024),
                                            ptx::sdesc_sw128(sSbar + kk * 2048, kHalfBytes, 1024), id_qs,
                                            kk > 0);
                            }
                        }
                        // MMA4: S += K^T V (K = the block's tokens; both operands MN-major)
#pragma unroll
                        for (int kk = 0; kk < kBlk / 16; ++kk) {
                            ptx::mma_ss(tmem + kColState, ptx::sdesc_sw128(sk + roff + kk * 2048, kHalfBytes, 1024),
                                        ptx::sdesc_sw128(sv + roff + kk * 2048, kHalfBytes, 1024), id_kv,
                                        (kk > 0 || has_state) ? 1u : 0u);
                        }
                        ptx::mma_commit(bar(ctrl->state_done));
                        if (sb == nsub - 1) ptx::mma_commit(bar(ctrl->k_empty[s]));   // K read
                        if (!ptx::mbar_wait(bar(ctrl->p_ready), n_blk & 1, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
                        // MMA2: O += P V (intra-block, left product); P from TMEM
#pragma unroll
                        for (int kk = 0; kk < kBlk / 16; ++kk) {
                            ptx::mma_ts(tmem + kColO, tmem + (kBlk == 128 ? p_col(kk) : p_col64(kk)),
                                        ptx::sdesc_sw128(sv + roff + kk * 2048, kHalfBytes, 1024), id_pv,
                                        (kk > 0 || has_state) ? 1u : 0u);
                        }
                        ptx::mma_commit(bar(ctrl->o_full));
                        has_state = true;
                        issued = true;
                    }
                    if (!ok) break;
                    ptx::mma_commit(bar(ctrl->empty[s]));
                }
                if (!ok) break;
                release_pos(pos);
                cur = nxi;
            }
            // teardown: every MMA this thread issued has completed
            if (issued) {
                ptx::mma_commit(bar(ctrl->drain));
                ptx::mbar_drain(bar(ctrl->drain), 0);
            }
        }
    } else if (warp < kFirstChainWarp) {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - kFirstEpiWarp; // 0..7
        const int sp = warp & 3;             // TMEM sub-partition this warp may access
        const int r = sp * 32 + lane;        // tile row owned by this thread
        const int k0 = 64 * (ew >> 2);       // score columns (keys) [k0, k0 + 64) of that row
        constexpr int kCols = kNV / 2;       // value columns per thread
        const int c0 = kCols * (ew >> 2);    // value columns [c0, c0 + kCols) of this part
        const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
        uint8_t* sbar_tile = smem + kSbarOffT;
        const bool store_leader = (ew == 0 && lane == 0);
        uint32_t n_blk = 0, n_tile = 0;
        // tile counter of the producer (phase A and phase C tiles), to know the
        // stage a phase-C block occupies
        uint32_t g = 0;
        auto n_tiles = [&](const Item& x) { return (uint32_t)((x.t1 - x.t0 + kTileRows - 1) / kTileRows); };
        bool ok = true;
        uint32_t pos = 0;
        int cur = n_items;
        if (!read_pos(0, cur)) ok = false;
        if (ok && cur < n_items) {
            const Item first = get_item(p, cur);
            if (has_phase_a(first)) g += n_tiles(first);
        }
        for (; ok && cur < n_items; ++pos) {
            const Item it = get_item(p, cur);
            int nxi = n_items;
            if (!read_pos(pos + 1, nxi)) { ok = false; break; }
            if (nxi < n_items) {
                const Item nx = get_item(p, nxi);
                if (has_phase_a(nx)) g += n_tiles(nx);
            }
            for (int t = it.t0; t < it.t1; t += kTileRows, ++g, ++n_tile) {
                const int s = g & 1;
                const int nsub = (kSub == 1 || it.t1 - t > kBlk) ? kSub : 1;
                const bool last_tile = t + kTileRows >= it.t1;
                // the last tile of a packed sequence is stored row by row, so that
                // the next sequence's rows are untouched
                const bool rowwise = packed && t + kTileRows > it.t1;
                uint8_t* ostage = smem + s * kStageB;
                // this thread's row in a block's M = kBlk accumulators: row r for
                // 128-token blocks; 16 sp + lane (lanes 0-15) for 64-token blocks
                const int br = (kBlk == 128) ? r : 16 * sp + lane;
                const bool row_ok = (kBlk == 128) || lane < 16;
                for (int sb = 0; sb < nsub; ++sb, ++n_blk) {
                    const bool last_block = last_tile && sb == nsub - 1;
                    const int trow = sb * kBlk + br;       // row within the 128-row tile
                    // ---- 1. P = tril(scores) as bf16 pairs over the first half of the
                    //         score columns this thread reads
                    if (!ptx::mbar_wait(bar(ctrl->s_full), n_blk & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    if constexpr (kBlk == 128) {
                        uint32_t pk[32];
                        if (k0 > sp * 32 + 31) {
                            // every key of this half lies above the diagonal for these rows
#pragma unroll
                            for (int j = 0; j < 32; ++j) pk[j] = 0u;
                        } else {
                            uint32_t v[64];
                            ptx::tmem_ld32(tl + kColS + k0, *reinterpret_cast<uint32_t(*)[32]>(v));
                            ptx::tmem_ld32(tl + kColS + k0 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                            ptx::tmem_ld_wait();
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int key = k0 + 2 * j;
                                const float a = (key <= r) ? __uint_as_float(v[2 * j]) : 0.0f;
                                const float b = (key + 1 <= r) ? __uint_as_float(v[2 * j + 1]) : 0.0f;
                                pk[j] = ptx::pack_bf16x2(a, b);
                            }
                        }
                        ptx::tmem_st32(tl + kColS + k0, pk);
                    } else {
                        // 64 x 64 scores: warpgroup h takes keys [32h, 32h+32)
                        const int kp0 = k0 >> 1;
                        uint32_t pk[16];
                        if (kp0 > 16 * sp + 15) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) pk[j] = 0u;
                        } else {
                            uint32_t v[32];
                            ptx::tmem_ld32(tl + kColS + kp0, v);
                            ptx::tmem_ld_wait();
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int key = kp0 + 2 * j;
                                const float a = (key <= br) ? __uint_as_float(v[2 * j]) : 0.0f;
                                const float b = (key + 1 <= br) ? __uint_as_float(v[2 * j + 1]) : 0.0f;
                                pk[j] = ptx::pack_bf16x2(a, b);
                            }
                        }
                        ptx::tmem_st16(tl + kColS + kp0, pk);
                    }
                    ptx::tmem_st_wait();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(ctrl->p_ready));

                    // ---- 2. state: bf16 copy for the next block, or the final state
                    if (!ptx::mbar_wait(bar(ctrl->state_done), n_blk & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    float* final_dst = nullptr;
                    if (last_block && p.state_out != nullptr && (!fused || it.last))
                        final_dst = p.state_out + (size_t)it.sidx * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim +
                                    it.vp * kNV + c0;
                    if (!last_block || final_dst != nullptr) {
                        uint32_t v[kCols];
#pragma unroll
                        for (int q = 0; q < kCols / 32; ++q)
                            ptx::tmem_ld32(tl + kColState + c0 + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * q));
                        ptx::tmem_ld_wait();
                        if (!last_block) {
#pragma unroll
                            for (int q = 0; q < kCols / 32; ++q) store_row32_bf16_sw128(sbar_tile, r, c0 + 32 * q, v + 32 * q);
                        } else {
                            float4* dst = reinterpret_cast<float4*>(final_dst);
#pragma unroll
                            for (int j = 0; j < kCols / 4; ++j)
                                dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                        }
                    }
                    ptx::tc_fence_before();
                    if (!last_block) {
                        ptx::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(bar(ctrl->sbar_ready));
                    } else {
                        // TMEM S and S̄ are no longer read for this item: the chain
                        // warps may write the next item's starting state
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(bar(ctrl->state_free));
                    }

                    // ---- 3. O: load to registers, release the accumulator, convert to
                    //         bf16 into the Q slot of this tile's stage (the block's
                    //         MMA1 and MMA3 have completed; a 64-token block's rows
                    //         do not overlap the rows the other block still reads)
                    if (!ptx::mbar_wait(bar(ctrl->o_full), n_blk & 1, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    {
                        uint32_t v[kCols];
#pragma unroll
                        for (int q = 0; q < kCols / 32; ++q)
                            ptx::tmem_ld32(tl + kColO + c0 + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * q));
                        ptx::tmem_ld_wait();
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(bar(ctrl->o_free));
                        if (!rowwise) {
                            if (row_ok) {
#pragma unroll
                                for (int q = 0; q < kCols / 32; ++q) store_row32_bf16_sw128(ostage, trow, c0 + 32 * q, v + 32 * q);
                            }
                            ptx::fence_proxy_async_smem();
                        } else if (row_ok && t + trow < it.t1) {
                            uint4* orow = reinterpret_cast<uint4*>(
                                p.o + ((size_t)it.z * p.rows + t + trow) * kHeadDim + it.vp * kNV + c0);
#pragma unroll
                            for (int j = 0; j < kCols / 8; ++j) {
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
                if (!ok) break;
                // ---- the tile's O rows are staged: one thread stores them with TMA
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(ctrl->o_staged));
                if (store_leader) {
                    if (!ptx::mbar_wait(bar(ctrl->o_staged), n_tile & 1, abort_flag)) { ok = false; }
                    if (ok && !rowwise) {
                        const uint32_t src = sbase + s * kStageB;
#pragma unroll
                        for (int hv = 0; hv < kVHalves; ++hv)
                            ptx::tma_store_3d(&maps.o, src + hv * kHalfBytes, it.vp * kNV + 64 * hv, t, it.z);
                        ptx::bulk_commit_group();
                        ptx::bulk_wait_group_read0();
                    }
                    ptx::mbar_arrive(bar(ctrl->o_stored[s]));
                }
                __syncwarp();
                if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) release_pos(pos);
            cur = nxi;
        }
        if (store_leader) ptx::bulk_wait_group0();
    } else {
        // ------------------------------------------------------------ chain warps
        // Starting state of every item; in the single pass also phase B.  Each
        // chain warp owns rows [32 sp, 32 sp + 32) of the state (a 16 KiB slice
        // with its own "published" flag), so the slices advance independently.
        // Phase B of an item runs while the epilogue is still on the previous
        // item; only writing the starting state waits for that item to finish.
        const int cw = warp - kFirstChainWarp;  // 0..3
        const int sp = warp & 3;
        const int r = sp * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
        uint8_t* sbar_tile = smem + kSbarOffT;
        uint32_t n_delta = 0, n_sf = 0;
        bool ok = true;
        bool first_item = true;
        for (uint32_t pos = 0; ok; ++pos) {
            int item = n_items;
            if (!read_pos(pos, item)) { ok = false; break; }
            if (item >= n_items) break;
            const Item it = get_item(p, item);
            const bool phase_a = has_phase_a(it);
            const bool look = fused && it.c > 0;
            const size_t roff = (size_t)r * kHeadDim + it.vp * kNV;   // row r, this value part
            const float* src = nullptr;          // exclusive prefix (with state_in)
            if (look) {
                src = p.chain + (size_t)(it.ws - 1) * (kHeadDim * kHeadDim) + roff;
            } else {
                const float* st0 = start_state(p, it);
                if (st0 != nullptr) src = st0 + roff;
            }
            const size_t fl = ((size_t)it.ws * p.vparts + it.vp) * kChainWarps + cw;   // own flag
            const size_t fl_prev = fl - (size_t)p.vparts * kChainWarps;               // chunk c-1's
            if (phase_a) {
                if (!ptx::mbar_wait(bar(ctrl->delta_done), n_delta++ & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
            }
            if (look) {
                // ---- wait for this slice of chunk c-1's inclusive prefix
                const int* f = p.flags + fl_prev;
                const unsigned long long t0 = globaltimer_ns();
                bool seen = false;
                while (true) {
                    const int v = ptx::ld_acquire_gpu(f);
                    if (__all_sync(0xffffffffu, v != 0)) { seen = true; break; }
                    if (*abort_flag) break;
                    if (globaltimer_ns() - t0 > wait_limit_ns()) {
                        *abort_flag = 1;
                        record_device_error(LA_ERR_TIMEOUT);
                        break;
                    }
                }
                if (!__all_sync(0xffffffffu, seen)) { ok = false; break; }
            }
            if (phase_a) {
                // ---- publish this slice of chunk c's inclusive prefix, 64 columns
                //      per round trip to L2
                float4* dst = reinterpret_cast<float4*>(p.chain + (size_t)it.ws * (kHeadDim * kHeadDim) + roff);
#pragma unroll
                for (int hh = 0; hh < kVHalves; ++hh) {
                    float pr[64];
                    if (src != nullptr) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float4 x = __ldcg(reinterpret_cast<const float4*>(src + 64 * hh) + j);
                            pr[4 * j + 0] = x.x;
                            pr[4 * j + 1] = x.y;
                            pr[4 * j + 2] = x.z;
                            pr[4 * j + 3] = x.w;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) pr[j] = 0.f;
                    }
#pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2) {
                        uint32_t d[32];
                        ptx::tmem_ld32(tl + kColDelta + 64 * hh + 32 * q2, d);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            __stcg(dst + 16 * hh + 8 * q2 + j,
                                   make_float4(pr[32 * q2 + 4 * j + 0] + __uint_as_float(d[4 * j + 0]),
                                               pr[32 * q2 + 4 * j + 1] + __uint_as_float(d[4 * j + 1]),
                                               pr[32 * q2 + 4 * j + 2] + __uint_as_float(d[4 * j + 2]),
                                               pr[32 * q2 + 4 * j + 3] + __uint_as_float(d[4 * j + 3])));
                    }
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) ptx::st_release_gpu(p.flags + fl, 1);
                // the increment has been read: TMEM is free for the next phase A
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(ctrl->delta_free));
            }
            // ---- starting state of phase C, once the previous item is done with it
            if (!first_item && !ptx::mbar_wait(bar(ctrl->state_free), n_sf++ & 1, abort_flag)) { ok = false; break; }
            first_item = false;
            ptx::tc_fence_after();
            if (src != nullptr) {
#pragma unroll
                for (int hh = 0; hh < kVHalves; ++hh) {
                    uint32_t f[64];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float4 x = look ? __ldcg(reinterpret_cast<const float4*>(src + 64 * hh) + j)
                                              : __ldg(reinterpret_cast<const float4*>(src + 64 * hh) + j);
                        f[4 * j + 0] = __float_as_uint(x.x);
                        f[4 * j + 1] = __float_as_uint(x.y);
                        f[4 * j + 2] = __float_as_uint(x.z);
                        f[4 * j + 3] = __float_as_uint(x.w);
                    }
                    ptx::tmem_st32(tl + kColState + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(f));
                    ptx::tmem_st32(tl + kColState + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(f + 32));
                    store_row32_bf16_sw128(sbar_tile, r, 64 * hh, f);
                    store_row32_bf16_sw128(sbar_tile, r, 64 * hh + 32, f + 32);
                }
                if (look) {
                    // this slice of chunk c-1's prefix has exactly one reader: drop it
#pragma unroll
                    for (int j = 0; j < kNV / 32; ++j) ptx::discard_l2_line(src + 32 * j);
                }
                ptx::tmem_st_wait();
                ptx::fence_proxy_async_smem();
            }
            ptx::tc_fence_before();
            __syncwarp();
            // sbar_ready counts epilogue warps: each chain warp stands for two
            if (lane == 0) ptx::mbar_arrive_cnt(bar(ctrl->sbar_ready), kEpiWarps / kChainWarps);
            if (lane == 0) release_pos(pos);
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
// Sequential kernel for split value columns (64 per CTA).
//
// One work item is a whole sequence (or a chunk of the three-pass schedule)
// for one half of the value columns.  The block loop is pipelined so that the
// tensor cores never wait for the epilogue:
//   * the state increment of each block, dS_i = K_i^T V_i, goes to one TMEM
//     buffer; the running state S (fp32) lives in the epilogue's registers (32
//     values per thread), which add dS_i and write the bf16 copy S̄_i for the
//     next block's Q S̄ into one of two shared-memory buffers;
//   * scores / P are double-buffered in TMEM and the output accumulator is
//     triple-buffered, so that Q S̄ of block i (the first product into O) waits
//     for the epilogue to have read the output of block i - 3, not i - 2: the
//     epilogue drains a block's output last in its turn of the next block.
// One issuing thread's MMAs complete one after another, about 175 cycles
// each whatever their shape (B200), while those of different threads
// overlap, so each product has its own issuing warp: A QK^T (MMA1), B Q S̄
// (MMA3), C P V (MMA2), D K^T V (MMA4), 8 MMAs per block each.
// V is last read by P V, the end of the block's dependency chain (QK^T -> P
// -> P V), so V has three slots of its own while Q and K share two stages:
// the load of block i + 3's V waits only for P V of block i.  Block i reads
// S̄ buffer i & 1; the state step of block i writes buffer (i + 1) & 1 once Q
// S̄ of block i - 1 has completed.  TMEM: scores 2 x 128, O 3 x 64, dS 64
// columns.  Shared memory: two stages of Q and K (128 x 128), three V slots
// (128 x 64), S̄ 2 x 16 KiB, O staging 16 KiB.
// ============================================================================
namespace sq {
constexpr int kNV = 64;
constexpr int kStageB = 2 * kTileBytes;                     // Q, K: 64 KiB
constexpr int kVSlots = 3;
constexpr int kVOff = kStages * kStageB;                    // V[3], 16 KiB each
constexpr int kSbarOff = kVOff + kVSlots * kHalfBytes;      // S̄[2], 16 KiB each
constexpr int kOstOff = kSbarOff + 2 * kHalfBytes;          // O staging, 16 KiB
constexpr int kCtrlOff = kOstOff + kHalfBytes;
constexpr int kSmemBytes = kCtrlOff + 512 + 1024;
constexpr uint32_t kColSP = 0;      // scores / P: 2 x 128
constexpr int kOBufs = 3;           // O accumulators: block g uses g % 3
constexpr uint32_t kColO = 256;     // output: 3 x 64
constexpr uint32_t kColDS = 448;    // state increment: 1 x 64
constexpr uint32_t kTmemCols = 512;
// Warp w runs on SM sub-partition w % 4 and its epilogue work is on TMEM lanes
// [32 (w % 4), +32).  Under the causal mask the P conversion of sub-partition
// i covers i + 1 chunks of 32 keys, and a warp issuing MMAs takes issue slots
// from the warps beside it, so the issuers sit on the sub-partitions with the
// least P work: A and C on 0, D on 1 (with the producer), B on 2, and only the
// store warp on 3.  Warps 2-9 form the epilogue, two per sub-partition.
constexpr int kEpiWarps = 8;
constexpr int kMmaAWarp = 0;                // issuer A: Q K^T
constexpr int kProducerWarp = 1;            // TMA loads; allocates TMEM
constexpr int kMmaBWarp = 2 + kEpiWarps;    // issuer B: Q S̄
constexpr int kStoreWarp = 3 + kEpiWarps;   // TMA stores of the staged O tiles
constexpr int kMmaCWarp = 4 + kEpiWarps;    // issuer C: P V
constexpr int kMmaDWarp = 5 + kEpiWarps;    // issuer D: K^T V
constexpr int kThreads = 32 * (6 + kEpiWarps);
constexpr int kL2Ahead = 2;                 // tiles prefetched into L2 ahead of the load

struct Ctrl {
    uint64_t full_qk[kStages];  // Q and K of stage s landed (MMA1 and MMA3 need no V)
    uint64_t full_v[kVSlots];   // V of slot v landed (packed tails: foreign rows cleared)
    uint64_t empty[kStages];    // Q and K slots of stage s read (A, B, D)
    uint64_t v_empty[kVSlots];  // V slot v read (C, D)
    uint64_t tail_ld;
    uint64_t s_full[2];     // MMA1 complete (scores buffer b)
    uint64_t p_ready[2];    // P of block parity b written (8 warps)
    uint64_t ds_full;       // MMA4 complete (the dS buffer)
    uint64_t p_free[2];     // MMA2 complete: P buffer b consumed
    uint64_t mma3_done[2];  // MMA3 (or, without a state, MMA1) of the block using buffer b
    uint64_t ds_free;       // dS buffer read (8 warps)
    uint64_t sbar_ready[2]; // S̄ read by the block of parity b written (8 warps)
    uint64_t o_full[kOBufs]; // MMA2 of a block using O buffer g % 3 complete
    uint64_t o_free[kOBufs]; // O buffer read (8 warps)
    uint64_t o_staged;      // O staged in shared memory (8 warps)
    uint64_t ost_free;      // the O staging buffer has been read by its TMA store
    uint64_t drain;         // teardown: every MMA of the four issuers complete
    uint32_t tmem_base;
    int abort;
};
}  // namespace sq

// kRev: the anti-causal form o_t = sum_{s >= t} (q_t . k_s) v_s (dense, one
// chunk per sequence): tiles are taken from the last to the first and the
// intra-block mask keeps keys at or after the row.  A template parameter, so
// that the causal instantiation carries none of it.
template <bool kRev>
__global__ void __launch_bounds__(sq::kThreads, 1)
prefill_seq_kernel(const __grid_constant__ TileMaps maps,
                   const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    sq::Ctrl* ctrl = reinterpret_cast<sq::Ctrl*>(smem + sq::kCtrlOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t sSbar = sbase + sq::kSbarOff;
    auto bar = [&](uint64_t& b) { return ptx::smem_u32(&b); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(ctrl->full_qk[s]), 1);
            ptx::mbar_init(bar(ctrl->empty[s]), 3);
        }
        for (int v = 0; v < sq::kVSlots; ++v) {
            ptx::mbar_init(bar(ctrl->full_v[v]), 1);
            ptx::mbar_init(bar(ctrl->v_empty[v]), 2);
        }
        ptx::mbar_init(bar(ctrl->ost_free), 1);
        ptx::mbar_init(bar(ctrl->tail_ld), 1);
        ptx::mbar_init(bar(ctrl->drain), 4);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(bar(ctrl->p_ready[b]), sq::kEpiWarps);
            ptx::mbar_init(bar(ctrl->sbar_ready[b]), sq::kEpiWarps);
        }
        for (int ob = 0; ob < sq::kOBufs; ++ob) {
            ptx::mbar_init(bar(ctrl->o_full[ob]), 1);
            ptx::mbar_init(bar(ctrl->o_free[ob]), sq::kEpiWarps);
        }
        ptx::mbar_init(bar(ctrl->o_staged), sq::kEpiWarps);
        ptx::mbar_init(bar(ctrl->ds_full), 1);
        ptx::mbar_init(bar(ctrl->ds_free), sq::kEpiWarps);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(bar(ctrl->s_full[b]), 1);
            ptx::mbar_init(bar(ctrl->p_free[b]), 1);
            ptx::mbar_init(bar(ctrl->mma3_done[b]), 1);
        }
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&ctrl->tmem_base), sq::kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&maps.q);
        ptx::prefetch_tmap(&maps.k);
        ptx::prefetch_tmap(&maps.v);
        ptx::prefetch_tmap(&maps.v_half);
        ptx::prefetch_tmap(&maps.o);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile int* abort_flag = &ctrl->abort;
    const int n_items = num_items(p);
    const bool packed = p.mode == kModeVarlen;
    const int stride = gridDim.x;
    // Row of the tile processed at step t (t = it.t0, it.t0 + 128, ...): the
    // same in the causal form; from the last tile back in the anti-causal one
    auto tile_row = [&](const Item& it, int t) {
        if constexpr (kRev) return it.t0 + ((it.t1 - it.t0 - 1) / kTileRows) * kTileRows - (t - it.t0);
        else return t;
    };

    if (warp == sq::kProducerWarp) {
        // ------------------------------------------------------------ producer
        // the other CTA of the head reads the same Q and K: normal L2 priority
        // for them, evict-first for this CTA's own V half
        const uint64_t pol_qk = ptx::policy_evict_normal();
        const uint64_t pol_v = ptx::policy_evict_first();
        uint32_t g = 0, n_tail = 0;
        bool ok = true;
        // the last loads issued into each stage and V slot (barrier, phase parity),
        // to let them land after an abort
        uint32_t ld_qk0 = 0, ld_qk1 = 0, par_qk0 = 0, par_qk1 = 0;
        uint32_t ld_v0 = 0, ld_v1 = 0, ld_v2 = 0, par_v0 = 0, par_v1 = 0, par_v2 = 0;
        // L2 prefetch of the tile `ahead` tiles after row t of the item (the
        // loads into shared memory then find it there)
        auto prefetch = [&](const Item& it, int t, int ahead) {
            const int tp = t + ahead * kTileRows;
            if (lane == 0 && tp < it.t1) {
                const int row = tile_row(it, tp);
                ptx::tma_prefetch_4d(&maps.q, 0, row, 0, it.z);
                ptx::tma_prefetch_4d(&maps.k, 0, row, 0, it.z);
                ptx::tma_prefetch_3d(&maps.v_half, it.vp * sq::kNV, row, it.z);
            }
        };
        for (int item = blockIdx.x; ok && item < n_items; item += stride) {
            const Item it = get_item(p, item);
            for (int j = 1; j < sq::kL2Ahead; ++j) prefetch(it, it.t0, j);
            for (int t = it.t0; ok && t < it.t1; t += kTileRows, ++g) {
                const int s = g & 1;
                const int vs = g % sq::kVSlots;
                const uint32_t stage = sbase + s * sq::kStageB;
                const uint32_t vslot = sbase + sq::kVOff + vs * kHalfBytes;
                prefetch(it, t, sq::kL2Ahead);
                // Q and K of block g reuse the stage that block g-2's MMA1, MMA3 and
                // MMA4 have finished with; V reuses the slot of block g-3, freed by
                // its MMA2 and MMA4
                const bool tail = packed && it.t1 - t < kTileRows;
                const uint32_t fv = tail ? bar(ctrl->tail_ld) : bar(ctrl->full_v[vs]);
                // test hook: this tile's loads stay unissued, so the waits for them
                // run out and the kernel aborts
                if (g + 1 == (uint32_t)p.stall_tile) continue;
                int w = 1;
                if (lane == 0) {
                    if (g >= 2) w = ptx::mbar_wait(bar(ctrl->empty[s]), ((g >> 1) + 1) & 1, abort_flag);
                    if (w) {
                        const int row = tile_row(it, t);
                        const uint32_t fqk = bar(ctrl->full_qk[s]);
                        ptx::mbar_arrive_expect_tx(fqk, 2 * kTileBytes);
                        ptx::tma_load_4d(stage, &maps.q, fqk, 0, row, 0, it.z, pol_qk);
                        ptx::tma_load_4d(stage + kTileBytes, &maps.k, fqk, 0, row, 0, it.z, pol_qk);
                        if (s) { ld_qk1 = fqk; par_qk1 = (g >> 1) & 1; }
                        else   { ld_qk0 = fqk; par_qk0 = (g >> 1) & 1; }
                        if (g >= sq::kVSlots)
                            w = ptx::mbar_wait(bar(ctrl->v_empty[vs]), ((g / sq::kVSlots) + 1) & 1, abort_flag);
                        if (w) {
                            ptx::mbar_arrive_expect_tx(fv, kHalfBytes);
                            ptx::tma_load_3d(vslot, &maps.v_half, fv, it.vp * sq::kNV, row, it.z, pol_v);
                            const uint32_t pv = tail ? (n_tail & 1) : ((g / sq::kVSlots) & 1);
                            if (vs == 0)      { ld_v0 = fv; par_v0 = pv; }
                            else if (vs == 1) { ld_v1 = fv; par_v1 = pv; }
                            else              { ld_v2 = fv; par_v2 = pv; }
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                if (tail) {
                    // a packed tail: clear the next sequence's rows of V, then release
                    if (lane == 0) w = ptx::mbar_wait(bar(ctrl->tail_ld), n_tail & 1, abort_flag);
                    ++n_tail;
                    if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                    zero_tail_rows(smem + sq::kVOff + vs * kHalfBytes, it.t1 - t, lane, 1);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(ctrl->full_v[vs]));
                }
            }
        }
        if (lane == 0) {
            for (uint32_t j = (g >= 2 ? g - 2 : 0); ok && j < g; ++j)
                ok = ptx::mbar_wait(bar(ctrl->empty[j & 1]), (j >> 1) & 1, abort_flag);
            for (uint32_t j = (g >= sq::kVSlots ? g - sq::kVSlots : 0); ok && j < g; ++j)
                ok = ptx::mbar_wait(bar(ctrl->v_empty[j % sq::kVSlots]), (j / sq::kVSlots) & 1, abort_flag);
            if (!ok) {
                // after an abort: let the loads already issued land (bounded)
                if (ld_qk0) ptx::mbar_drain(ld_qk0, par_qk0);
                if (ld_qk1) ptx::mbar_drain(ld_qk1, par_qk1);
                if (ld_v0) ptx::mbar_drain(ld_v0, par_v0);
                if (ld_v1) ptx::mbar_drain(ld_v1, par_v1);
                if (ld_v2) ptx::mbar_drain(ld_v2, par_v2);
            }
        }
    } else if (warp == sq::kMmaAWarp || warp == sq::kMmaBWarp || warp == sq::kMmaCWarp || warp == sq::kMmaDWarp) {
        // ------------------------------------------------------------ MMA issuers
        // A: MMA1 scores = Q K^T; B: MMA3 O = Q S̄; C: MMA2 O += P V; D: MMA4
        // dS = K^T V.  Every resource one of them reuses is buffered (scores / P
        // and S̄ by block parity b, O by g % 3, dS once) and guarded by a
        // barrier of that buffer.
        if (lane == 0) {
            constexpr uint32_t id_qk = ptx::idesc_bf16(128, 128, false, false);  // Q K^T
            constexpr uint32_t id_qs = ptx::idesc_bf16(128, sq::kNV, false, true);   // Q S̄
            constexpr uint32_t id_kv = ptx::idesc_bf16(128, sq::kNV, true, true);    // K^T V
            constexpr uint32_t id_pv = ptx::idesc_bf16(128, sq::kNV, false, true);   // P V
            const int role = warp == sq::kMmaAWarp ? 0 : warp == sq::kMmaBWarp ? 1 : warp == sq::kMmaCWarp ? 2 : 3;
            uint32_t g = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += stride) {
                const Item it = get_item(p, item);
                bool has_state = start_state(p, it) != nullptr;
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    const int s = g & 1;
                    const uint32_t b = g & 1;
                    const uint32_t par = (g >> 1) & 1;           // phase parity of buffer b's barriers
                    const uint32_t prev = ((g >> 1) + 1) & 1;    // ... for block g - 2
                    const int vs = g % sq::kVSlots;
                    if (role != 2 && !ptx::mbar_wait(bar(ctrl->full_qk[s]), par, abort_flag)) { ok = false; break; }
                    if (role >= 2 && !ptx::mbar_wait(bar(ctrl->full_v[vs]), (g / sq::kVSlots) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sq_ = sbase + s * sq::kStageB;
                    const uint32_t sk = sq_ + kTileBytes;
                    const uint32_t sv = sbase + sq::kVOff + vs * kHalfBytes;
                    const uint32_t ob = g % sq::kOBufs;
                    const uint32_t o_cols = tmem + sq::kColO + ob * sq::kNV;
                    if (role == 0) {
                        // MMA1 into scores buffer b, once MMA2 of block g-2 consumed its P
                        if (g >= 2 && !ptx::mbar_wait(bar(ctrl->p_free[b]), prev, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                            ptx::mma_ss(tmem + sq::kColSP + b * 128, ptx::sdesc_sw128(sq_ + off, 16, 1024),
                                        ptx::sdesc_sw128(sk + off, 16, 1024), id_qk, kk > 0);
                        }
                        ptx::mma_commit(bar(ctrl->s_full[b]));
                        ptx::mma_commit(bar(ctrl->empty[s]));
                    } else if (role == 1) {
                        // MMA3: O = Q S̄_{g-1} (S̄ buffer g & 1) into O buffer g % 3, once
                        // that S̄ is written and the epilogue has read block g-3's O there
                        if (!ptx::mbar_wait(bar(ctrl->sbar_ready[b]), par, abort_flag)) { ok = false; break; }
                        if (g >= sq::kOBufs &&
                            !ptx::mbar_wait(bar(ctrl->o_free[ob]), ((g / sq::kOBufs) + 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        if (has_state) {
                            const uint32_t sb = sSbar + (g & 1) * kHalfBytes;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                                ptx::mma_ss(o_cols, ptx::sdesc_sw128(sq_ + off, 16, 1024),
                                            ptx::sdesc_sw128(sb + kk * 2048, kHalfBytes, 1024), id_qs, kk > 0);
                            }
                        }
                        ptx::mma_commit(bar(ctrl->mma3_done[b]));
                        ptx::mma_commit(bar(ctrl->empty[s]));
                    } else if (role == 3) {
                        // MMA4: dS = K^T V, once the state step has read block g-1's dS
                        if (g >= 1 && !ptx::mbar_wait(bar(ctrl->ds_free), (g - 1) & 1, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            ptx::mma_ss(tmem + sq::kColDS, ptx::sdesc_sw128(sk + kk * 2048, kHalfBytes, 1024),
                                        ptx::sdesc_sw128(sv + kk * 2048, kHalfBytes, 1024), id_kv, kk > 0);
                        ptx::mma_commit(bar(ctrl->ds_full));
                        ptx::mma_commit(bar(ctrl->empty[s]));      // K read
                        ptx::mma_commit(bar(ctrl->v_empty[vs]));   // V read by MMA4
                    } else {
                        // MMA2: O += P V (P in TMEM buffer b), after MMA3 wrote O
                        if (!ptx::mbar_wait(bar(ctrl->p_ready[b]), par, abort_flag)) { ok = false; break; }
                        if (!ptx::mbar_wait(bar(ctrl->mma3_done[b]), par, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            ptx::mma_ts(o_cols, tmem + sq::kColSP + b * 128 + p_col(kk) - kColS,
                                        ptx::sdesc_sw128(sv + kk * 2048, kHalfBytes, 1024), id_pv,
                                        (kk > 0 || has_state) ? 1u : 0u);
                        ptx::mma_commit(bar(ctrl->o_full[ob]));
                        ptx::mma_commit(bar(ctrl->p_free[b]));
                        ptx::mma_commit(bar(ctrl->v_empty[vs]));   // V read by MMA2
                    }
                    has_state = true;
                }
            }
            // teardown: every MMA the four issuers issued has completed
            ptx::mma_commit(bar(ctrl->drain));
            ptx::mbar_drain(bar(ctrl->drain), 0);
        }
    } else if (warp == sq::kStoreWarp) {
        // ------------------------------------------------------------ O stores
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += stride) {
                const Item it = get_item(p, item);
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    if (!ptx::mbar_wait(bar(ctrl->o_staged), g & 1, abort_flag)) { ok = false; break; }
                    if (!(packed && t + kTileRows > it.t1)) {
                        ptx::tma_store_3d(&maps.o, sbase + sq::kOstOff, it.vp * sq::kNV, tile_row(it, t), it.z);
                        ptx::bulk_commit_group();
                        ptx::bulk_wait_group_read0();
                    }
                    ptx::mbar_arrive(bar(ctrl->ost_free));
                }
            }
            ptx::bulk_wait_group0();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Per block g: P(g), then S += dS_g and S̄_g, then the output of the
        // PREVIOUS block, so that MMA2(g) (issued once P(g) is written) runs
        // while this block's state and the previous output are handled.
        const int ew = warp - 2;             // 0..7
        const int sp = warp & 3;             // TMEM sub-partition of this warp
        const int r = sp * 32 + lane;        // tile row owned by this thread
        const int k0 = 64 * (ew >> 2);       // keys [k0, k0 + 64) for P
        const int c0 = 32 * (ew >> 2);       // value columns [c0, c0 + 32) of this part
        const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
        uint32_t g = 0;
        bool ok = true;
        // Arrive on sbar_ready for block gb.  Eight warps arrive once per block,
        // so a warp two blocks ahead of a slower one could complete the slower
        // one's phase in its place.  It cannot get there: a warp reaches the
        // state step of block g only after MMA4(g), which waits for every warp's
        // ds_free of block g - 1, and each warp arrives on ds_free only after
        // its S̄ arrival of that step (below).
        auto sbar_arrive = [&](uint32_t gb) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->sbar_ready[gb & 1]));
        };
        // the block whose output is still to be drained
        bool o_pending = false;
        Item o_it;
        int o_t = 0;
        uint32_t o_g = 0;
        // ---- O of block og: registers, release its buffer, stage as bf16 for
        //      the store warp once it has stored the previous tile
        auto drain_o = [&](const Item& oit, int ot, uint32_t og) -> bool {
            const uint32_t ob = og % sq::kOBufs;
            if (!ptx::mbar_wait(bar(ctrl->o_full[ob]), (og / sq::kOBufs) & 1, abort_flag)) return false;
            ptx::tc_fence_after();
            const bool rowwise = packed && ot + kTileRows > oit.t1;
            uint8_t* ostage = smem + sq::kOstOff;
            uint32_t v[32];
            ptx::tmem_ld32(tl + sq::kColO + ob * sq::kNV + c0, v);
            ptx::tmem_ld_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->o_free[ob]));
            if (og >= 1 && !ptx::mbar_wait(bar(ctrl->ost_free), (og - 1) & 1, abort_flag)) return false;
            if (!rowwise) {
                store_row32_bf16_sw128(ostage, r, c0, v);
                ptx::fence_proxy_async_smem();
            } else if (ot + r < oit.t1) {
                uint4* orow = reinterpret_cast<uint4*>(
                    p.o + ((size_t)oit.z * p.rows + ot + r) * kHeadDim + oit.vp * sq::kNV + c0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 w;
                    w.x = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
                    w.y = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
                    w.z = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
                    w.w = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
                    orow[j] = w;
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->o_staged));
            return true;
        };
        for (int item = blockIdx.x; ok && item < n_items; item += stride) {
            const Item it = get_item(p, item);
            const int vcol = it.vp * sq::kNV + c0;  // first owned column of the 128
            // ---- running state S (row r, columns vcol..vcol+31) and S̄ for block g
            //      (S̄ buffer g & 1, last read by MMA3 of block g - 2, whose output
            //      this warp has drained)
            float srun[32];
            if (const float* st0 = start_state(p, it)) {
                const float4* src = reinterpret_cast<const float4*>(st0 + (size_t)r * kHeadDim + vcol);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 x = __ldg(src + j);
                    srun[4 * j + 0] = x.x;
                    srun[4 * j + 1] = x.y;
                    srun[4 * j + 2] = x.z;
                    srun[4 * j + 3] = x.w;
                }
                uint32_t f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) f[j] = __float_as_uint(srun[j]);
                store_row32_bf16_sw128(smem + sq::kSbarOff + (g & 1) * kHalfBytes, r, c0, f);
                ptx::fence_proxy_async_smem();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) srun[j] = 0.f;
            }
            sbar_arrive(g);

            for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                const bool last_block = t + kTileRows >= it.t1;
                const uint32_t b = g & 1;
                // ---- 1. P = tril(scores) as bf16 pairs, in place in buffer b
                if (!ptx::mbar_wait(bar(ctrl->s_full[b]), (g >> 1) & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    // keys [kq, kq + 32), packed into columns [k0 + 16 q2, +16): the
                    // second half's store lands on columns the first half has read.
                    // The warp's rows are [32 sp, 32 sp + 32): a chunk wholly on the
                    // kept side of the diagonal is packed as is, one wholly on the
                    // other side is zero (not loaded), only kq = 32 sp is masked.
                    const int kq = k0 + 32 * q2;
                    const uint32_t scol = tl + sq::kColSP + b * 128 + kq;
                    const bool none = kRev ? (kq < sp * 32) : (kq > sp * 32);
                    const bool all = kRev ? (kq > sp * 32) : (kq < sp * 32);
                    uint32_t pk[16];
                    if (none) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[j] = 0u;
                    } else {
                        uint32_t v[32];
                        ptx::tmem_ld32(scol, v);
                        ptx::tmem_ld_wait();
                        if (all) {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                pk[j] = ptx::pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                        } else {
                            // the diagonal chunk: keys kq + i against row kq + lane
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const bool keep_a = kRev ? 2 * j >= lane : 2 * j <= lane;
                                const bool keep_b = kRev ? 2 * j + 1 >= lane : 2 * j + 1 <= lane;
                                const float a = keep_a ? __uint_as_float(v[2 * j]) : 0.0f;
                                const float bb = keep_b ? __uint_as_float(v[2 * j + 1]) : 0.0f;
                                pk[j] = ptx::pack_bf16x2(a, bb);
                            }
                        }
                    }
                    ptx::tmem_st16(tl + sq::kColSP + b * 128 + k0 + 16 * q2, pk);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(ctrl->p_ready[b]));

                // ---- 2. S += dS_g; S̄_g for the next block, or the final state
                if (!ptx::mbar_wait(bar(ctrl->ds_full), g & 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                {
                    uint32_t d[32];
                    ptx::tmem_ld32(tl + sq::kColDS + c0, d);
                    ptx::tmem_ld_wait();
                    ptx::tc_fence_before();
#pragma unroll
                    for (int j = 0; j < 32; ++j) srun[j] += __uint_as_float(d[j]);
                }
                if (!last_block) {
                    // S̄ buffer (g + 1) & 1, last read by MMA3 of block g - 1.  Its phase
                    // cannot run ahead: MMA3 of block g + 1 needs the S̄ written here.
                    if (g >= 1 && !ptx::mbar_wait(bar(ctrl->mma3_done[(g + 1) & 1]), ((g - 1) >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint32_t f[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) f[j] = __float_as_uint(srun[j]);
                    store_row32_bf16_sw128(smem + sq::kSbarOff + ((g + 1) & 1) * kHalfBytes, r, c0, f);
                    ptx::fence_proxy_async_smem();
                    sbar_arrive(g + 1);
                } else if (p.state_out != nullptr) {
                    float4* dst = reinterpret_cast<float4*>(
                        p.state_out + (size_t)it.sidx * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim + vcol);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_float4(srun[4 * j], srun[4 * j + 1], srun[4 * j + 2], srun[4 * j + 3]);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(ctrl->ds_free));

                // ---- 3. the previous block's output
                if (o_pending && !drain_o(o_it, o_t, o_g)) { ok = false; break; }
                o_pending = true;
                o_it = it;
                o_t = t;
                o_g = g;
            }
        }
        if (ok && o_pending) drain_o(o_it, o_t, o_g);
    }


    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, sq::kTmemCols);
    }
}

// ============================================================================
// Sequential kernel for split value columns (64 per CTA) with 64-token blocks.
//
// Each 128-row tile is processed as two 64-token blocks h = 0, 1 (rows
// [64 h, 64 h + 64)):
//     O_h = Q_h S̄_{h-1} + tril(Q_h K_h^T)^bf16 V_h          (M = 64 MMAs)
//     S_h = S_{h-1} + K_h^T V_h                               (M = 128, K = 64)
// so the state is updated, and rounded to bf16 for the inter-block product,
// every 64 tokens.  The M = 64 accumulators (scores / P, O) hold row m in TMEM
// lane 32 (m / 16) + m % 16: lanes 0-15 of each 32-lane sub-partition.
// A block takes 8 (Q K^T) + 8 (Q S̄) + 4 (K^T V) + 4 (P V) MMA instructions,
// 48 per tile.  One issuing thread's MMAs complete one after another, about
// 175 cycles each whatever their shape (B200), while the MMAs of different
// issuing threads overlap, so four warps issue them: A the scores (MMA1), B
// the inter-block products (MMA3), C P V (MMA2) and D the state increments
// (MMA4).  D depends on nothing but the loads, so the state chain (dS -> S̄
// -> Q S̄) never waits behind a P V that waits for Q S̄.
// Every buffer is indexed by the block's position h in its tile and each of
// its barriers completes once per tile, so phase parity = tile & 1.
// TMEM: scores / P 2 x 64, O 2 x 64 (M = 64 layout), dS 2 x 64 columns.
// Shared memory: two stages of Q and K, three V slots (64 columns; V is
// last read by P V, the end of the chain), two S̄ buffers of 16 KiB (block h
// of a tile reads buffer h; the state step writes the other one once Q S̄ of
// the previous block has completed) and O staging.
// ============================================================================
namespace sq64 {
constexpr int kNV = 64;
constexpr int kStageB = 2 * kTileBytes;                     // Q, K: 64 KiB
constexpr int kVSlots = 3;
constexpr int kVOff = kStages * kStageB;                    // V[3]
constexpr int kSbarOff = kVOff + kVSlots * kHalfBytes;      // S̄[2]
constexpr int kOstOff = kSbarOff + 2 * kHalfBytes;
constexpr int kCtrlOff = kOstOff + kHalfBytes;
constexpr int kSmemBytes = kCtrlOff + 512 + 1024;
constexpr uint32_t kColSP = 0;      // scores / P: 2 x 64
constexpr uint32_t kColO = 128;     // output: 2 x 64
constexpr uint32_t kColDS = 256;    // state increment: 2 x 64
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiWarps = 8;
constexpr int kStoreWarp = 2 + kEpiWarps;   // TMA stores of the staged O tiles
constexpr int kMmaBWarp = 3 + kEpiWarps;    // issuer B: Q S̄
constexpr int kMmaCWarp = 4 + kEpiWarps;    // issuer C: P V
constexpr int kMmaDWarp = 5 + kEpiWarps;    // issuer D: K^T V
constexpr int kThreads = 32 * (6 + kEpiWarps);
constexpr int kL2Ahead = 2;
constexpr uint32_t kRowOff = 64 * 128;      // row 64 of a 128B-swizzled 64-column half

// Column, within a scores buffer, of the bf16 P pairs for keys [16 kk, 16 kk +
// 16): the warp that converts keys [32 w, 32 w + 32) packs them into the first
// 16 of the 32 columns it read.
__host__ __device__ constexpr uint32_t p_col(int kk) { return kk < 2 ? kk * 8 : 32 + (kk - 2) * 8; }

struct Ctrl {
    uint64_t full_qk[kStages];  // Q and K of stage s landed
    uint64_t full_v[kVSlots];   // V of slot v landed (packed tails: foreign rows cleared)
    uint64_t empty[kStages];    // Q and K slots read: one commit each from A, B and D
    uint64_t v_empty[kVSlots];  // V slot read: one commit each from C and D
    uint64_t tail_ld;
    uint64_t s_full[2];     // MMA1 of block h complete
    uint64_t p_ready[2];    // P of block h written (8 warps)
    uint64_t pv_done[2];    // MMA2 of block h complete: P consumed, O final
    uint64_t ds_full[2];    // MMA4 of block h complete
    uint64_t ds_free[2];    // dS of block h read (8 warps)
    uint64_t mma3_done[2];  // MMA3 of block h complete (or none needed)
    uint64_t sbar_ready[2]; // S̄ read by block h written (8 warps)
    uint64_t o_free[2];     // O of block h read (8 warps)
    uint64_t o_staged;      // both blocks of a tile staged (8 warps)
    uint64_t ost_free;      // the staging buffer has been read by its TMA store
    uint64_t drain;         // teardown: every MMA of the four issuers complete
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Ctrl) <= 512, "control block");
}  // namespace sq64

__global__ void __launch_bounds__(sq64::kThreads, 1)
prefill_seq64_kernel(const __grid_constant__ TileMaps maps,
                     const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    sq64::Ctrl* ctrl = reinterpret_cast<sq64::Ctrl*>(smem + sq64::kCtrlOff);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t sSbar = sbase + sq64::kSbarOff;
    auto bar = [&](uint64_t& b) { return ptx::smem_u32(&b); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(ctrl->full_qk[s]), 1);
            ptx::mbar_init(bar(ctrl->empty[s]), 3);
        }
        for (int v = 0; v < sq64::kVSlots; ++v) {
            ptx::mbar_init(bar(ctrl->full_v[v]), 1);
            ptx::mbar_init(bar(ctrl->v_empty[v]), 2);
        }
        ptx::mbar_init(bar(ctrl->tail_ld), 1);
        ptx::mbar_init(bar(ctrl->o_staged), sq64::kEpiWarps);
        ptx::mbar_init(bar(ctrl->ost_free), 1);
        ptx::mbar_init(bar(ctrl->drain), 4);
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(bar(ctrl->s_full[b]), 1);
            ptx::mbar_init(bar(ctrl->p_ready[b]), sq64::kEpiWarps);
            ptx::mbar_init(bar(ctrl->pv_done[b]), 1);
            ptx::mbar_init(bar(ctrl->ds_full[b]), 1);
            ptx::mbar_init(bar(ctrl->ds_free[b]), sq64::kEpiWarps);
            ptx::mbar_init(bar(ctrl->mma3_done[b]), 1);
            ptx::mbar_init(bar(ctrl->sbar_ready[b]), sq64::kEpiWarps);
            ptx::mbar_init(bar(ctrl->o_free[b]), sq64::kEpiWarps);
        }
        ctrl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&ctrl->tmem_base), sq64::kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&maps.q);
        ptx::prefetch_tmap(&maps.k);
        ptx::prefetch_tmap(&maps.v_half);
        ptx::prefetch_tmap(&maps.o);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile int* abort_flag = &ctrl->abort;
    const int n_items = num_items(p);
    const bool packed = p.mode == kModeVarlen;
    const int stride = gridDim.x;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_qk = ptx::policy_evict_normal();   // shared with the other half
        const uint64_t pol_v = ptx::policy_evict_first();
        uint32_t g = 0, n_tail = 0;
        bool ok = true;
        // the last loads issued into each stage, barrier and phase parity, to let
        // them land after an abort
        uint32_t ld_qk0 = 0, ld_qk1 = 0, ld_v0 = 0, ld_v1 = 0;
        uint32_t par_qk0 = 0, par_qk1 = 0, par_v0 = 0, par_v1 = 0;
        auto prefetch = [&](const Item& it, int t, int ahead) {
            const int tp = t + ahead * kTileRows;
            if (lane == 0 && tp < it.t1) {
                ptx::tma_prefetch_4d(&maps.q, 0, tp, 0, it.z);
                ptx::tma_prefetch_4d(&maps.k, 0, tp, 0, it.z);
                ptx::tma_prefetch_3d(&maps.v_half, it.vp * sq64::kNV, tp, it.z);
            }
        };
        for (int item = blockIdx.x; ok && item < n_items; item += stride) {
            const Item it = get_item(p, item);
            for (int j = 1; j < sq64::kL2Ahead; ++j) prefetch(it, it.t0, j);
            for (int t = it.t0; ok && t < it.t1; t += kTileRows, ++g) {
                const int s = g & 1;
                const int vs = g % sq64::kVSlots;
                const uint32_t stage = sbase + s * sq64::kStageB;
                const uint32_t vslot = sbase + sq64::kVOff + vs * kHalfBytes;
                prefetch(it, t, sq64::kL2Ahead);
                const bool tail = packed && it.t1 - t < kTileRows;
                const uint32_t fv = tail ? bar(ctrl->tail_ld) : bar(ctrl->full_v[vs]);
                // test hook: this tile's loads stay unissued, so the waits for them
                // run out and the kernel aborts
                if (g + 1 == (uint32_t)p.stall_tile) continue;
                int w = 1;
                if (lane == 0) {
                    if (g >= 2) w = ptx::mbar_wait(bar(ctrl->empty[s]), ((g >> 1) + 1) & 1, abort_flag);
                    if (w) {
                        const uint32_t fqk = bar(ctrl->full_qk[s]);
                        ptx::mbar_arrive_expect_tx(fqk, 2 * kTileBytes);
                        ptx::tma_load_4d(stage, &maps.q, fqk, 0, t, 0, it.z, pol_qk);
                        ptx::tma_load_4d(stage + kTileBytes, &maps.k, fqk, 0, t, 0, it.z, pol_qk);
                        if (s) { ld_qk1 = fqk; par_qk1 = (g >> 1) & 1; }
                        else   { ld_qk0 = fqk; par_qk0 = (g >> 1) & 1; }
                        if (g >= sq64::kVSlots)
                            w = ptx::mbar_wait(bar(ctrl->v_empty[vs]), ((g / sq64::kVSlots) + 1) & 1, abort_flag);
                        if (w) {
                            ptx::mbar_arrive_expect_tx(fv, kHalfBytes);
                            ptx::tma_load_3d(vslot, &maps.v_half, fv, it.vp * sq64::kNV, t, it.z, pol_v);
                            const uint32_t pv = tail ? (n_tail & 1) : ((g / sq64::kVSlots) & 1);
                            if (s) { ld_v1 = fv; par_v1 = pv; }
                            else   { ld_v0 = fv; par_v0 = pv; }
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                if (tail) {
                    if (lane == 0) w = ptx::mbar_wait(bar(ctrl->tail_ld), n_tail & 1, abort_flag);
                    ++n_tail;
                    if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                    zero_tail_rows(smem + sq64::kVOff + vs * kHalfBytes, it.t1 - t, lane, 1);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(ctrl->full_v[vs]));
                }
            }
        }
        if (lane == 0) {
            for (uint32_t j = (g >= 2 ? g - 2 : 0); ok && j < g; ++j)
                ok = ptx::mbar_wait(bar(ctrl->empty[j & 1]), (j >> 1) & 1, abort_flag);
            for (uint32_t j = (g >= sq64::kVSlots ? g - sq64::kVSlots : 0); ok && j < g; ++j)
                ok = ptx::mbar_wait(bar(ctrl->v_empty[j % sq64::kVSlots]), (j / sq64::kVSlots) & 1, abort_flag);
            if (!ok) {
                // after an abort: let the loads already issued land (bounded)
                if (ld_qk0) ptx::mbar_drain(ld_qk0, par_qk0);
                if (ld_qk1) ptx::mbar_drain(ld_qk1, par_qk1);
                if (ld_v0) ptx::mbar_drain(ld_v0, par_v0);
                if (ld_v1) ptx::mbar_drain(ld_v1, par_v1);
            }
        }
    } else if (warp == 1 || warp == sq64::kMmaBWarp || warp == sq64::kMmaCWarp || warp == sq64::kMmaDWarp) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            constexpr uint32_t id_qk = ptx::idesc_bf16(64, 64, false, false);        // Q_h K_h^T
            constexpr uint32_t id_qs = ptx::idesc_bf16(64, sq64::kNV, false, true);  // Q_h S̄
            constexpr uint32_t id_kv = ptx::idesc_bf16(128, sq64::kNV, true, true);  // K_h^T V_h
            constexpr uint32_t id_pv = ptx::idesc_bf16(64, sq64::kNV, false, true);  // P_h V_h
            const int role = warp == 1 ? 0 : warp == sq64::kMmaBWarp ? 1 : warp == sq64::kMmaCWarp ? 2 : 3;
            uint32_t g = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += stride) {
                const Item it = get_item(p, item);
                bool has_state = start_state(p, it) != nullptr;
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    const int s = g & 1;
                    const uint32_t tp = g & 1;        // this tile's phase of the block barriers
                    const uint32_t pp = tp ^ 1u;      // the previous tile's
                    if (!ptx::mbar_wait(bar(ctrl->full_qk[s]), (g >> 1) & 1, abort_flag)) { ok = false; break; }
                    const int vs = g % sq64::kVSlots;
                    if (role >= 2 && !ptx::mbar_wait(bar(ctrl->full_v[vs]), (g / sq64::kVSlots) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sq_ = sbase + s * sq64::kStageB;
                    const uint32_t sk = sq_ + kTileBytes;
                    const uint32_t sv = sbase + sq64::kVOff + vs * kHalfBytes;
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t roff = h * sq64::kRowOff;
                        if (role == 0) {
                            // MMA1: scores_h = Q_h K_h^T, once MMA2 of block h of the
                            // previous tile has consumed the P in buffer h
                            if (g >= 1 && !ptx::mbar_wait(bar(ctrl->pv_done[h]), pp, abort_flag)) { ok = false; break; }
                            ptx::tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32 + roff;
                                ptx::mma_ss(tmem + sq64::kColSP + h * 64, ptx::sdesc_sw128(sq_ + off, 16, 1024),
                                            ptx::sdesc_sw128(sk + off, 16, 1024), id_qk, kk > 0);
                            }
                            ptx::mma_commit(bar(ctrl->s_full[h]));
                        } else if (role == 1) {
                            // MMA3: O_h = Q_h S̄ (S̄ buffer h), once that S̄
                            // is written and block h of the previous tile has been drained
                            if (!ptx::mbar_wait(bar(ctrl->sbar_ready[h]), tp, abort_flag)) { ok = false; break; }
                            if (g >= 1 && !ptx::mbar_wait(bar(ctrl->o_free[h]), pp, abort_flag)) { ok = false; break; }
                            ptx::tc_fence_after();
                            if (has_state) {
                                const uint32_t sb = sSbar + h * kHalfBytes;
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk) {
                                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32 + roff;
                                    ptx::mma_ss(tmem + sq64::kColO + h * 64, ptx::sdesc_sw128(sq_ + off, 16, 1024),
                                                ptx::sdesc_sw128(sb + kk * 2048, kHalfBytes, 1024), id_qs, kk > 0);
                                }
                            }
                            ptx::mma_commit(bar(ctrl->mma3_done[h]));
                        } else if (role == 3) {
                            // MMA4: dS_h = K_h^T V_h, once dS buffer h has been read
                            if (g >= 1 && !ptx::mbar_wait(bar(ctrl->ds_free[h]), pp, abort_flag)) { ok = false; break; }
                            ptx::tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                ptx::mma_ss(tmem + sq64::kColDS + h * 64,
                                            ptx::sdesc_sw128(sk + roff + kk * 2048, kHalfBytes, 1024),
                                            ptx::sdesc_sw128(sv + roff + kk * 2048, kHalfBytes, 1024), id_kv, kk > 0);
                            ptx::mma_commit(bar(ctrl->ds_full[h]));
                        } else {
                            // MMA2: O_h += P_h V_h (P from TMEM), after MMA3 wrote O_h
                            if (!ptx::mbar_wait(bar(ctrl->p_ready[h]), tp, abort_flag)) { ok = false; break; }
                            if (!ptx::mbar_wait(bar(ctrl->mma3_done[h]), tp, abort_flag)) { ok = false; break; }
                            ptx::tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                ptx::mma_ts(tmem + sq64::kColO + h * 64, tmem + sq64::kColSP + h * 64 + sq64::p_col(kk),
                                            ptx::sdesc_sw128(sv + roff + kk * 2048, kHalfBytes, 1024), id_pv,
                                            (kk > 0 || has_state) ? 1u : 0u);
                            ptx::mma_commit(bar(ctrl->pv_done[h]));
                            if (h == 1) ptx::mma_commit(bar(ctrl->v_empty[vs]));  // V read
                        }
                        has_state = true;
                    }
                    if (!ok) break;
                    if (role != 2) ptx::mma_commit(bar(ctrl->empty[s]));     // Q and K read
                    if (role == 3) ptx::mma_commit(bar(ctrl->v_empty[vs]));  // V read by MMA4
                }
            }
            // teardown: every MMA the three issuers issued has completed
            ptx::mma_commit(bar(ctrl->drain));
            ptx::mbar_drain(bar(ctrl->drain), 0);
        }
    } else if (warp == sq64::kStoreWarp) {
        // ------------------------------------------------------------ O stores
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int item = blockIdx.x; ok && item < n_items; item += stride) {
                const Item it = get_item(p, item);
                for (int t = it.t0; t < it.t1; t += kTileRows, ++g) {
                    if (!ptx::mbar_wait(bar(ctrl->o_staged), g & 1, abort_flag)) { ok = false; break; }
                    if (!(packed && t + kTileRows > it.t1)) {
                        ptx::tma_store_3d(&maps.o, sbase + sq64::kOstOff, it.vp * sq64::kNV, t, it.z);
                        ptx::bulk_commit_group();
                        ptx::bulk_wait_group_read0();
                    }
                    ptx::mbar_arrive(bar(ctrl->ost_free));
                }
            }
            ptx::bulk_wait_group0();
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Per block (g, h): P, then S += dS and S̄ for the next block, then the
        // output of the previous block.
        const int ew = warp - 2;             // 0..7
        const int sp = warp & 3;             // TMEM sub-partition of this warp
        const int r = sp * 32 + lane;        // state row (key dimension) of this thread
        const int c0 = 32 * (ew >> 2);       // keys [c0, c0 + 32) of P; value columns
                                             // [c0, c0 + 32) of S and O (of this CTA's 64)
        // P and O of a 64-token block (M = 64 layout, rows in lanes 0-15): thread
        // lane takes row 16 sp + (lane & 15) and 16 of the warp's 32 columns,
        // [c0 + 16 (lane >> 4), +16)
        const int br = 16 * sp + (lane & 15);
        const int cq = c0 + 16 * (lane >> 4);
        const uint32_t tl = tmem + ((uint32_t)(sp * 32) << 16);
        uint8_t* ostage = smem + sq64::kOstOff;
        uint32_t g = 0;
        bool ok = true;
        // Arrive on sbar_ready[x] for tile gt.  A warp running ahead of a slower
        // one cannot complete the slower one's phase: it reaches the next state
        // step of block position h only after MMA4 of that block, which waits for
        // every warp's ds_free of the same position a tile earlier, and each warp
        // arrives on ds_free only after its S̄ arrival of that step.
        auto sbar_arrive = [&](int x) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->sbar_ready[x]));
        };
        bool o_pending = false;
        Item o_it;
        int o_t = 0, o_h = 0;
        uint32_t o_g = 0;
        // ---- O of block (og, oh): registers, release its buffer, stage as bf16
        //      (the tile's staging buffer once the previous tile has been stored)
        auto drain_o = [&](const Item& oit, int ot, uint32_t og, int oh) -> bool {
            if (!ptx::mbar_wait(bar(ctrl->pv_done[oh]), og & 1, abort_flag)) return false;
            ptx::tc_fence_after();
            const bool rowwise = packed && ot + kTileRows > oit.t1;
            uint32_t v[16];
            ptx::tmem_ld16x2_16<16>(tl + sq64::kColO + oh * 64 + c0, v);
            ptx::tmem_ld_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(ctrl->o_free[oh]));
            if (oh == 0 && og >= 1 && !ptx::mbar_wait(bar(ctrl->ost_free), (og - 1) & 1, abort_flag)) return false;
            const int trow = 64 * oh + br;
            if (!rowwise) {
                store_row16_bf16_sw128(ostage, trow, cq, v);
                ptx::fence_proxy_async_smem();
            } else if (ot + trow < oit.t1) {
                uint4* orow = reinterpret_cast<uint4*>(
                    p.o + ((size_t)oit.z * p.rows + ot + trow) * kHeadDim + oit.vp * sq64::kNV + cq);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint4 w;
                    w.x = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
                    w.y = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
                    w.z = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
                    w.w = ptx::pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
                    orow[j] = w;
                }
            }
            __syncwarp();
            if (oh == 1 && lane == 0) ptx::mbar_arrive(bar(ctrl->o_staged));
            return true;
        };
        for (int item = blockIdx.x; ok && item < n_items; item += stride) {
            const Item it = get_item(p, item);
            const int vcol = it.vp * sq64::kNV + c0;   // first owned column of the 128
            // ---- running state S (row r, columns vcol..vcol+31) and the S̄ of the
            //      item's first block (buffer 0, last read by MMA3 of block 0 of the
            //      previous tile, whose output this warp has drained)
            float srun[32];
            if (const float* st0 = start_state(p, it)) {
                const float4* src = reinterpret_cast<const float4*>(st0 + (size_t)r * kHeadDim + vcol);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 x = __ldg(src + j);
                    srun[4 * j + 0] = x.x;
                    srun[4 * j + 1] = x.y;
                    srun[4 * j + 2] = x.z;
                    srun[4 * j + 3] = x.w;
                }
                uint32_t f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) f[j] = __float_as_uint(srun[j]);
                store_row32_bf16_sw128(smem + sq64::kSbarOff, r, c0, f);
                ptx::fence_proxy_async_smem();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) srun[j] = 0.f;
            }
            sbar_arrive(0);

            for (int t = it.t0; ok && t < it.t1; t += kTileRows, ++g) {
                const bool last_tile = t + kTileRows >= it.t1;
                const uint32_t tp = g & 1;
                for (int h = 0; h < 2; ++h) {
                    // ---- 1. P_h = tril(scores_h) as bf16 pairs, in place
                    if (!ptx::mbar_wait(bar(ctrl->s_full[h]), tp, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    {
                        // keys [cq, cq + 16) of row br; packed into columns [c0, c0 + 8)
                        // (threads 0-15) and [c0 + 8, c0 + 16) (threads 16-31)
                        const uint32_t scol = tl + sq64::kColSP + h * 64 + c0;
                        uint32_t pk[8];
                        if (c0 > 16 * sp + 15) {
                            // every key of the warp's 32 lies above the diagonal for its rows
#pragma unroll
                            for (int j = 0; j < 8; ++j) pk[j] = 0u;
                        } else {
                            uint32_t v[16];
                            ptx::tmem_ld16x2_16<16>(scol, v);
                            ptx::tmem_ld_wait();
                            if (c0 + 31 <= 16 * sp) {
                                // every key at or below every row of the warp
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    pk[j] = ptx::pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                            } else {
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const int key = cq + 2 * j;
                                    const float a = (key <= br) ? __uint_as_float(v[2 * j]) : 0.0f;
                                    const float b = (key + 1 <= br) ? __uint_as_float(v[2 * j + 1]) : 0.0f;
                                    pk[j] = ptx::pack_bf16x2(a, b);
                                }
                            }
                        }
                        ptx::tmem_st16x2_8<8>(scol, pk);
                    }
                    ptx::tmem_st_wait();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(ctrl->p_ready[h]));

                    // ---- 2. S += dS_h; S̄ for the next block, or the final state
                    if (!ptx::mbar_wait(bar(ctrl->ds_full[h]), tp, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    {
                        uint32_t d[32];
                        ptx::tmem_ld32(tl + sq64::kColDS + h * 64 + c0, d);
                        ptx::tmem_ld_wait();
                        ptx::tc_fence_before();
#pragma unroll
                        for (int j = 0; j < 32; ++j) srun[j] += __uint_as_float(d[j]);
                    }
                    if (!(last_tile && h == 1)) {
                        // S̄ for the next block: buffer h ^ 1, last read by MMA3 of the
                        // previous block, block 1 of the previous tile (h = 0) or block 0
                        // of this one (h = 1).  Its phase cannot run ahead: the next MMA3
                        // of that block position needs the S̄ written here.
                        if ((g >= 1 || h == 1) &&
                            !ptx::mbar_wait(bar(ctrl->mma3_done[h ^ 1]), h == 0 ? (tp ^ 1u) : tp, abort_flag)) {
                            ok = false;
                            break;
                        }
                        uint32_t f[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) f[j] = __float_as_uint(srun[j]);
                        store_row32_bf16_sw128(smem + sq64::kSbarOff + (h ^ 1) * kHalfBytes, r, c0, f);
                        ptx::fence_proxy_async_smem();
                        // block (g, 1) for h = 0, block (g + 1, 0) for h = 1
                        sbar_arrive(h ^ 1);
                    } else if (p.state_out != nullptr) {
                        float4* dst = reinterpret_cast<float4*>(
                            p.state_out + (size_t)it.sidx * (kHeadDim * kHeadDim) + (size_t)r * kHeadDim + vcol);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            dst[j] = make_float4(srun[4 * j], srun[4 * j + 1], srun[4 * j + 2], srun[4 * j + 3]);
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(bar(ctrl->ds_free[h]));

                    // ---- 3. the previous block's output
                    if (o_pending && !drain_o(o_it, o_t, o_g, o_h)) { ok = false; break; }
                    o_pending = true;
                    o_it = it;
                    o_t = t;
                    o_g = g;
                    o_h = h;
                }
            }
        }
        if (ok && o_pending) drain_o(o_it, o_t, o_g, o_h);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, sq64::kTmemCols);
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
chunk_state_kernel(const __grid_constant__ TileMaps maps,
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
        ptx::prefetch_tmap(&maps.k);
        ptx::prefetch_tmap(&maps.v);
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
                if (!produce_tile<false>(maps, smem + s * cs::kStageBytes,
                                         sbase + s * cs::kStageBytes, bar(ctrl->full[s]),
                                         bar(ctrl->tail_ld), n_tail, t, it.z, it.t1 - t, packed, pol,
                                         pol, lane, abort_flag)) {
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
chunk_scan_kernel(float* ws, float* state_out, int n_chunks, const float* state_in) {
    const int bh = blockIdx.y;
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;   // < 128*128
    float4 acc = state_in != nullptr
                     ? *reinterpret_cast<const float4*>(state_in + (size_t)bh * (kHeadDim * kHeadDim) + e)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
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
                         int H, int num_seqs, const float* state_in) {
    if (*seq_ok == 0) return;
    const int j = blockIdx.x;
    const int hh = blockIdx.y;
    const int total = chunk_off[num_seqs];
    const int c0 = chunk_off[j], c1 = chunk_off[j + 1];
    constexpr int kStride4 = kHeadDim * kHeadDim / 4;
    float4* base = reinterpret_cast<float4*>(ws + (size_t)hh * total * (kHeadDim * kHeadDim));
    const float4* in4 = state_in != nullptr
                            ? reinterpret_cast<const float4*>(state_in + ((size_t)j * H + hh) * (kHeadDim * kHeadDim))
                            : nullptr;
    for (int e4 = threadIdx.x; e4 < kStride4; e4 += blockDim.x) {
        float4 acc = in4 != nullptr ? in4[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
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

// Exclusive prefix over ranks of per-rank states (sequence parallelism): out =
// sum_{r < rank} states[r], summed in rank order.  states is [R][n4] float4.
__global__ void __launch_bounds__(256)
state_prefix_kernel(const float4* states, int rank, long n4, float4* out) {
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < rank; ++r) {
            const float4 x = states[(size_t)r * n4 + i];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        out[i] = acc;
    }
}

// Single pass over packed sequences: an empty sequence owns no work item, so
// its final state (its starting state, or zero) is written here.  Grid
// (num_seqs, H).
__global__ void __launch_bounds__(256)
zero_empty_states_kernel(float* state_out, const int32_t* cu, const int* seq_ok, int H,
                         const float* state_in) {
    if (*seq_ok == 0) return;
    const int j = blockIdx.x;
    if (cu[j + 1] != cu[j]) return;
    const size_t off = ((size_t)j * H + blockIdx.y) * (kHeadDim * kHeadDim);
    float4* dst = reinterpret_cast<float4*>(state_out + off);
    const float4* src = state_in != nullptr ? reinterpret_cast<const float4*>(state_in + off) : nullptr;
    for (int e = threadIdx.x; e < kHeadDim * kHeadDim / 4; e += blockDim.x)
        dst[e] = src != nullptr ? src[e] : make_float4(0.f, 0.f, 0.f, 0.f);
}

// cu_seqlens check and chunk offsets of packed sequences (one CTA): verdict in
// *ok, chunk_off[j] = sum over earlier sequences of ceil(len / chunk_tokens),
// chunk_off[num_seqs] = chunks per head.  A malformed array records
// LA_ERR_BAD_SEQLENS and yields zero chunks.  Check cu_seqlens and number the chunks of every sequence (chunk_off).  With
// `order` non-null (one chunk per sequence: chunk_tokens >= every length) it
// also lists the non-empty sequences longest first, ties by index: a
// persistent grid that walks items in that order takes the long ones first.
__global__ void varlen_prepare_kernel(const int32_t* cu, int num_seqs, int total, int chunk_tokens,
                                      int* ok, int32_t* chunk_off, int32_t* order) {
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
    if (order == nullptr) return;
    __syncthreads();
    if (bad) return;
    for (int j = threadIdx.x; j < num_seqs; j += blockDim.x) {
        const int len = cu[j + 1] - cu[j];
        if (len == 0) continue;
        int rank = 0;
        for (int i = 0; i < num_seqs; ++i) {
            const int li = cu[i + 1] - cu[i];
            rank += (li > len || (li == len && i < j)) ? 1 : 0;
        }
        order[rank] = j;   // empty sequences rank after every non-empty one
    }
}

}  // namespace tc
}  // namespace la
