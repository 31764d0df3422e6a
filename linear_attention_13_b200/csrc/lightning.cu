// lightning.cu -- the C ABI of liblightning.so (declared in include/lightning.h):
// argument validation, dispatch to the kernels, TMA descriptor creation,
// stream-ordered workspace, device status.  One translation unit holds every
// kernel so that the device status word needs no separate device link.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "lightning.h"
#include "common.cuh"
#include "ptx.cuh"
#include "prefill_tc.cuh"
#include "prefill_simt.cuh"
#include "tokens.cuh"
#include "decode.cuh"

namespace la {

// A CTA with most of an SM's shared memory that waits (bounded, on
// %globaltimer) and exits: la_debug_occupy_sms holds SMs away from other
// kernels with it, so that tests can run the look-back prefill on part of the
// GPU.  It waits on nothing but the clock.
constexpr int kOccupySmem = 160 * 1024;
__global__ void __launch_bounds__(32) occupy_kernel(unsigned long long duration_ns) {
    extern __shared__ uint8_t occupied[];
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < duration_ns) __nanosleep(2000);
    if (threadIdx.x == 0) occupied[0] = 0;
}

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    bool smem_attrs_set = false;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
int g_host_status = LA_OK;   // last asynchronous CUDA error seen by the host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Allocations that the next calls must fail, as if the stream-ordered pool
// were out of memory (la_debug_fail_allocations: host-side failure injection
// for the tests; zero in normal use).
std::atomic<int> g_fail_allocs{0};

// Every workspace of the library comes from here: stream-ordered memory on
// `s`.  Returns false (after clearing the CUDA error) when it cannot be had;
// the callers then return LA_ERR_ALLOC before launching anything.
bool ws_alloc(void** ptr, size_t bytes, cudaStream_t s) {
    int n = g_fail_allocs.load();
    while (n > 0) {
        if (g_fail_allocs.compare_exchange_weak(n, n - 1)) return false;
    }
    if (cudaMallocAsync(ptr, bytes, s) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return true;
}

int note_cuda(cudaError_t e) {
    if (e == cudaSuccess) return LA_OK;
    std::lock_guard<std::mutex> lk(g_mutex);
    if (g_host_status == LA_OK) g_host_status = LA_ERR_CUDA;
    return LA_ERR_CUDA;
}

// Per-device setup: SM count, kernel attributes, the driver entry point.
int device_setup(int* dev_out, int* sms_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mutex);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return LA_ERR_CUDA;
        if (cudaFuncSetAttribute(tc::prefill_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::smem_bytes(128)) != cudaSuccess ||
            cudaFuncSetAttribute(tc::prefill_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::smem_bytes(64)) != cudaSuccess ||
            cudaFuncSetAttribute(tc::prefill_tc_kernel<128, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::smem_bytes(128)) != cudaSuccess ||
            cudaFuncSetAttribute(tc::prefill_seq_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::sq::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(tc::prefill_seq_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::sq::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(tc::prefill_seq64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::sq64::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(tc::chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tc::cs::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(simt::prefill_simt_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 simt::smem_bytes<64>()) != cudaSuccess ||
            cudaFuncSetAttribute(simt::prefill_simt_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 simt::smem_bytes<128>()) != cudaSuccess ||
            cudaFuncSetAttribute(simt::prefill_simt_varlen_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 simt::smem_bytes<64>()) != cudaSuccess ||
            cudaFuncSetAttribute(simt::prefill_simt_varlen_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 simt::smem_bytes<128>()) != cudaSuccess ||
            cudaFuncSetAttribute(decode::decode_step_q8_kernel<__nv_bfloat16, 128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Q8Smem<128>::kBytes) != cudaSuccess ||
            cudaFuncSetAttribute(decode::decode_step_q8_kernel<__nv_bfloat16, 64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Q8Smem<64>::kBytes) != cudaSuccess ||
            cudaFuncSetAttribute(decode::decode_step_q8_kernel<float, 128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Q8Smem<128>::kBytes) != cudaSuccess ||
            cudaFuncSetAttribute(decode::decode_step_q8_kernel<float, 64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode::Q8Smem<64>::kBytes) != cudaSuccess) {
            cudaGetLastError();
            return LA_ERR_CUDA;
        }
        if (g_encode == nullptr) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                 cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                return LA_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        // Keep up to 2 GiB of freed workspace in the default stream-ordered pool
        // instead of returning it to the driver at every synchronisation.
        cudaMemPool_t pool;
        if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
            uint64_t keep = 2ull << 30;
            cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        }
        cudaGetLastError();
        di.sm_count = sms;
        di.ready = true;
    }
    *dev_out = dev;
    *sms_out = di.sm_count;
    return LA_OK;
}

// ------------------------------------------------------------ kernel timing
struct Timing {
    bool enabled = false;
    int cap = 0;
    int used = 0;
    std::vector<cudaEvent_t> ev;     // 2 * cap events (start, stop)
    std::vector<int> kid;            // kernel id of each used pair
    int launches[LA_NUM_KERNEL_IDS] = {0};
};
Timing g_timing;

void timing_release() {
    for (cudaEvent_t e : g_timing.ev) cudaEventDestroy(e);
    g_timing.ev.clear();
    g_timing.kid.clear();
    g_timing.cap = g_timing.used = 0;
    g_timing.enabled = false;
    for (int& c : g_timing.launches) c = 0;
}

// Record the start event of a launch of kernel `id` on `s`; returns the slot
// (or -1 when timing is off or the pool is full).
int timing_begin(int id, cudaStream_t s) {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_timing.enabled) return -1;
    g_timing.launches[id]++;
    if (g_timing.used >= g_timing.cap) return -1;
    const int slot = g_timing.used++;
    g_timing.kid[slot] = id;
    cudaEventRecord(g_timing.ev[2 * slot], s);
    return slot;
}

void timing_end(int slot, cudaStream_t s) {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_mutex);
    if (slot < g_timing.used) cudaEventRecord(g_timing.ev[2 * slot + 1], s);
}

// Brackets one kernel launch with timing events.
struct TimedLaunch {
    int slot;
    cudaStream_t s;
    TimedLaunch(int id, cudaStream_t st) : slot(timing_begin(id, st)), s(st) {}
    ~TimedLaunch() { timing_end(slot, s); }
};

// NVTX range named after a C entry point, around the whole host call (checks,
// descriptor set-up, launches), so that profiler timelines group the kernels
// by call.  A pointer test when no profiler is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D bf16 tensor map over [outer][rows][128] with a {64, 128, 1} box and the
// 128-byte swizzle; rows past `rows` read as zero.
// [outer][rows][128] bf16 as {64 columns, rows, 2 halves, outer}: a
// {64, 128, 2, 1} box is one whole tile in two 128B-swizzled halves.
int make_tmap_bf16_tile(CUtensorMap* m, const void* base, uint64_t rows, uint64_t outer) {
    cuuint64_t dims[4] = {64, (cuuint64_t)rows, 2, (cuuint64_t)outer};
    cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, 128, (cuuint64_t)rows * kHeadDim * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)kTileRows, 2, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LA_OK : LA_ERR_CUDA;
}

int make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t outer) {
    cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows, (cuuint64_t)outer};
    cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)rows * kHeadDim * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTileRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LA_OK : LA_ERR_CUDA;
}

int make_tile_maps(tc::TileMaps* m, const void* q, const void* k, const void* v, const void* o,
                   uint64_t rows, uint64_t outer) {
    if (make_tmap_bf16_tile(&m->q, q, rows, outer) || make_tmap_bf16_tile(&m->k, k, rows, outer) ||
        make_tmap_bf16_tile(&m->v, v, rows, outer) || make_tmap_bf16(&m->v_half, v, rows, outer) ||
        make_tmap_bf16(&m->o, o, rows, outer) || make_tmap_bf16(&m->k_half, k, rows, outer))
        return LA_ERR_CUDA;
    return LA_OK;
}

// Chunk length (tokens, multiple of 128) for the bf16 dense path: the
// makespan of ceil(items / CTAs) rounds of (blocks per chunk + per-chunk
// overhead) is minimised, with chunks of at least 512 tokens.
int choose_chunk_tokens(int BH, int N, int ctas) {
    const int nblk = (N + kTileRows - 1) / kTileRows;
    int best_blocks = nblk;
    double best_cost = 1e300;
    const int min_blocks = std::min(4, nblk);
    for (int cb = nblk; cb >= min_blocks; --cb) {
        const int nchunks = (nblk + cb - 1) / cb;
        if (nchunks > 1 && cb * (nchunks - 1) >= nblk) continue;
        const long items = (long)BH * nchunks;
        const long rounds = (items + ctas - 1) / ctas;
        const double cost = (double)rounds * (cb + 1.5) + (nchunks > 1 ? 3.0 : 0.0);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best_blocks = cb;
        }
    }
    return best_blocks * kTileRows;
}

// Main kernel for p.vparts value parts per head (1: 128 columns per CTA, 2: 64).
// Split value columns without a look-back chain run the sequential kernels
// with the fully double-buffered block pipeline (prefill_seq64_kernel for
// 64-token blocks); otherwise 64-token blocks run the 128-column kernel with
// two blocks per tile.
std::atomic<const char*> g_main_kernel{""};

// Tile (counted per CTA, plus one) whose loads the next split-kernel launch
// leaves unissued (la_debug_stall_split_load: a test hook), or 0.
std::atomic<int> g_stall_tile{0};

void launch_main(const tc::TileMaps& m, const tc::Params& p0, int grid, cudaStream_t stream) {
    tc::Params p = p0;
    if (p.vparts == 2 && !p.fused) p.stall_tile = g_stall_tile.exchange(0);
    if (p.blk == 64 && p.vparts == 2 && !p.fused) {
        g_main_kernel = "prefill_seq64_kernel";
        tc::prefill_seq64_kernel<<<grid, tc::sq64::kThreads, tc::sq64::kSmemBytes, stream>>>(m, p);
    } else if (p.blk == 64) {
        g_main_kernel = "prefill_tc_kernel<128,64>";
        tc::prefill_tc_kernel<128, 64><<<grid, tc::kThreads, tc::smem_bytes(128), stream>>>(m, p);
    } else if (p.vparts == 2 && !p.fused) {
        g_main_kernel = "prefill_seq_kernel";
        tc::prefill_seq_kernel<false><<<grid, tc::sq::kThreads, tc::sq::kSmemBytes, stream>>>(m, p);
    } else if (p.vparts == 2) {
        g_main_kernel = "prefill_tc_kernel<64>";
        tc::prefill_tc_kernel<64><<<grid, tc::kThreads, tc::smem_bytes(64), stream>>>(m, p);
    } else {
        g_main_kernel = "prefill_tc_kernel<128>";
        tc::prefill_tc_kernel<128><<<grid, tc::kThreads, tc::smem_bytes(128), stream>>>(m, p);
    }
}

tc::Params dense_params(int BH, int N, int chunk_tokens, void* o) {
    tc::Params p;
    std::memset(&p, 0, sizeof(p));
    p.mode = tc::kModeDense;
    p.Z = BH;
    p.rows = N;
    p.chunk_tokens = chunk_tokens;
    p.n_chunks = (N + chunk_tokens - 1) / chunk_tokens;
    p.n_items = BH * p.n_chunks;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.vparts = 1;
    p.blk = 128;
    return p;
}

// Split the value columns of every head over two CTAs when the heads alone
// would leave many SMs idle and the sequences are short enough that one CTA
// per (head, half) finishes in time (measured on B200: at 64 heads the split
// wins at 8K tokens and loses to chunking at 256K).
// When the split fills 80-100 % of the SMs with one CTA per (head, half), it
// also wins for long sequences: every tile is read once, where chunking reads
// the K and V of every chunk with a successor twice (B200, 64 heads of 262144
// tokens: 3.47 ms split against 3.95 ms for the best chunking).
bool want_split_v(long slices, long N, int sms, int flags) {
    if (flags & LA_FLAG_NO_SPLIT_V) return false;
    if (flags & LA_FLAG_SPLIT_V) return true;
    if (2 * slices * 5 >= (long)sms * 4 && 2 * slices <= (long)sms) return true;
    return slices * 4 < (long)sms * 3 && N <= 16384;
}

// chunk states -> scan -> outputs, with the chunk states in `ws`
void launch_three_pass(const tc::TileMaps& m, tc::Params p, float* ws, float* state_out, int grid,
                       cudaStream_t stream) {
    p.chunk_delta = ws;
    {
        // chunk states are computed once per chunk over all value columns
        tc::Params pc = p;
        pc.vparts = 1;
        pc.n_items = p.Z * p.n_chunks;
        TimedLaunch tl(LA_KERNEL_CHUNK_STATE, stream);
        tc::chunk_state_kernel<<<std::min(grid, pc.n_items), tc::cs::kThreads, tc::cs::kSmemBytes,
                                 stream>>>(m, pc);
    }
    {
        TimedLaunch tl(LA_KERNEL_CHUNK_SCAN, stream);
        dim3 sgrid(kHeadDim * kHeadDim / 4 / 256, p.Z);
        tc::chunk_scan_kernel<<<sgrid, 256, 0, stream>>>(ws, state_out, p.n_chunks, p.state_in);
    }
    p.prefix = ws;
    p.state_out = nullptr;
    {
        TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
        launch_main(m, p, grid, stream);
    }
}

// Chunk length for the single-pass schedule: minimise rounds of work items
// times the time of an item, in 128-token blocks: a chunk with a successor
// also reads its K and V once more for the look-back (half a block's bytes
// per block) and hands its prefix over (about two blocks).  Chunks of at least
// 512 tokens.
int choose_fused_chunk_tokens(int Z, int N, int ctas) {
    const int nblk = (N + kTileRows - 1) / kTileRows;
    int best = nblk;
    double best_cost = 1e300;
    for (int cb = nblk; cb >= std::min(4, nblk); --cb) {
        const int nch = (nblk + cb - 1) / cb;
        if (nch > 1 && cb * (nch - 1) >= nblk) continue;
        const long rounds = ((long)Z * nch + ctas - 1) / ctas;
        const double cost = (double)rounds * (nch > 1 ? 1.5 * cb + 2.0 : cb + 0.5);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = cb;
        }
    }
    return best * kTileRows;
}

// Items the next look-back launch skips (la_debug_skip_lookback_items: a test
// hook; their successors' bounded waits then run out).  Consumed by one launch.
std::atomic<int> g_skip_items{0};

// Single pass with look-back: one launch (plus a memset of the chunk flags and
// the item counter).
int launch_fused(const tc::TileMaps& m, tc::Params p,
                 long n_chunk_slots, float* state_out, int grid, cudaStream_t stream) {
    p.state_out = state_out;
    if (n_chunk_slots > 0) {
        const size_t chain_bytes = (size_t)n_chunk_slots * kHeadDim * kHeadDim * sizeof(float);
        const size_t flag_words = (size_t)n_chunk_slots * p.vparts * tc::kChainWarps + 1;  // + counter
        const size_t flag_bytes = (flag_words * sizeof(int) + 255) / 256 * 256;
        uint8_t* buf = nullptr;
        if (!ws_alloc(reinterpret_cast<void**>(&buf), chain_bytes + flag_bytes, stream)) {
            return LA_ERR_ALLOC;
        }
        p.flags = reinterpret_cast<int*>(buf);
        p.ticket = p.flags + flag_words - 1;
        p.ticket_base = g_skip_items.exchange(0);
        p.chain = reinterpret_cast<float*>(buf + flag_bytes);
        p.fused = 1;
        cudaMemsetAsync(p.flags, 0, flag_words * sizeof(int), stream);
        {
            TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
            launch_main(m, p, grid, stream);
        }
        const int st = note_cuda(cudaGetLastError());
        cudaFreeAsync(buf, stream);
        return st;
    }
    p.fused = 0;
    {
        TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
        launch_main(m, p, grid, stream);
    }
    return note_cuda(cudaGetLastError());
}

// The anti-causal form o_t = sum_{s >= t} (q_t . k_s) v_s, bf16, d = 128, 128-token
// blocks: prefill_seq_kernel with one chunk per sequence, walking its blocks from
// the last to the first (the state then holds suffix sums).  It runs when the
// sequences are short (N <= kReverseMaxN) or when one CTA pair per sequence
// fills the GPU (as the forward's split schedule); other shapes return
// LA_ERR_UNSUPPORTED: too few CTAs would each walk too many blocks.
constexpr int kReverseMaxN = 16384;

bool reverse_direct_ok(long BH, long N, int sms) {
    return N <= kReverseMaxN || (2 * BH * 5 >= (long)sms * 4 && 2 * BH <= (long)sms);
}

int launch_prefill_reverse_bf16(const void* q, const void* k, const void* v, void* o, int BH, int N,
                                cudaStream_t stream, int sms) {
    if (!reverse_direct_ok(BH, N, sms)) return LA_ERR_UNSUPPORTED;
    tc::TileMaps m;
    if (make_tile_maps(&m, q, k, v, o, N, BH)) return LA_ERR_CUDA;
    tc::Params p = dense_params(BH, N, ((N + kTileRows - 1) / kTileRows) * kTileRows, o);
    p.vparts = 2;
    p.blk = 128;
    p.n_items *= 2;
    const int grid = std::min(p.n_items, sms);
    {
        TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
        g_main_kernel = "prefill_seq_kernel<anti-causal>";
        tc::prefill_seq_kernel<true><<<grid, tc::sq::kThreads, tc::sq::kSmemBytes, stream>>>(m, p);
    }
    return note_cuda(cudaGetLastError());
}

int launch_prefill_bf16(const void* q, const void* k, const void* v, void* o, float* state_out,
                        int BH, int N, int blk, cudaStream_t stream, int sms, int chunk_tokens,
                        int flags, const float* state_in) {
    if (blk != 128 && blk != 64) return LA_ERR_UNSUPPORTED;
    tc::TileMaps m;
    if (make_tile_maps(&m, q, k, v, o, N, BH)) return LA_ERR_CUDA;
    const bool three_pass = (flags & LA_FLAG_THREE_PASS) != 0;
    int vparts = want_split_v(BH, N, sms, flags) ? 2 : 1;
    if (!three_pass) {
        const int asked = chunk_tokens;
        if (chunk_tokens <= 0) chunk_tokens = choose_fused_chunk_tokens(BH * vparts, N, sms);
        chunk_tokens = ((chunk_tokens + kTileRows - 1) / kTileRows) * kTileRows;
        if (blk == 64 && vparts == 2 && chunk_tokens < N) {
            // 64-token blocks split the value columns only in the sequential
            // kernel (one chunk per sequence); chunked, they keep whole rows
            vparts = 1;
            chunk_tokens = asked > 0 ? asked : choose_fused_chunk_tokens(BH, N, sms);
            chunk_tokens = ((chunk_tokens + kTileRows - 1) / kTileRows) * kTileRows;
        }
        tc::Params p = dense_params(BH, N, chunk_tokens, o);
        p.vparts = vparts;
        p.blk = blk;
        p.state_in = state_in;
        p.n_items *= vparts;
        const int grid = std::min(p.n_items, sms);
        return launch_fused(m, p, p.n_chunks > 1 ? (long)BH * p.n_chunks : 0, state_out,
                            grid, stream);
    }
    if (chunk_tokens <= 0) chunk_tokens = choose_chunk_tokens(BH * vparts, N, sms);
    chunk_tokens = ((chunk_tokens + kTileRows - 1) / kTileRows) * kTileRows;
    tc::Params p = dense_params(BH, N, chunk_tokens, o);
    p.vparts = vparts;
    p.blk = blk;
    p.state_in = state_in;
    p.n_items *= vparts;
    const int grid = std::min(p.n_items, sms);

    if (p.n_chunks == 1) {
        p.state_out = state_out;
        {
            TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
            launch_main(m, p, grid, stream);
        }
        return note_cuda(cudaGetLastError());
    }
    float* ws = nullptr;
    const size_t ws_bytes = (size_t)BH * p.n_chunks * kHeadDim * kHeadDim * sizeof(float);
    if (!ws_alloc(reinterpret_cast<void**>(&ws), ws_bytes, stream)) {
        return LA_ERR_ALLOC;
    }
    launch_three_pass(m, p, ws, state_out, grid, stream);
    int st = note_cuda(cudaGetLastError());
    cudaFreeAsync(ws, stream);
    return st;
}

// Single pass over packed sequences: chunks of about half a CTA's share of the
// work, H * T / (2 * ctas) tokens, at least 8192.  A chunk with a successor
// has its K and V read twice, so long chunks save traffic as long as the work
// items stay small against a CTA's share (B200, 2^20 tokens x 64 heads in
// sequences of 1K-64K tokens: 8192-token chunks 17.4 ms, one chunk per
// sequence 12.5 ms).
int choose_varlen_fused_chunk_tokens(int H, int T, int ctas) {
    const long share = (long)H * T / (2L * std::max(ctas, 1));
    const long t_rounded = ((long)T + kTileRows - 1) / kTileRows * kTileRows;
    return (int)std::max(8192L, std::min(share, t_rounded));
}

// Chunk length for packed sequences: long enough to keep the chunk-state
// traffic small, short enough for about eight rounds of work items.
int choose_varlen_chunk_tokens(int H, int T, int ctas) {
    long target = ((long)H * T) / (8L * ctas);
    target = std::max(1024L, std::min(16384L, target));
    return (int)(((target + kTileRows - 1) / kTileRows) * kTileRows);
}

// Packed sequences with the value columns of every (sequence, head) split over
// two CTAs and no chunking: one item per (sequence, head, half), longest
// sequences first, run by the sequential kernel.  Nothing is read twice.
int launch_prefill_varlen_split(const void* q, const void* k, const void* v, void* o,
                                float* state_out, const int32_t* cu_seqlens, int num_seqs, int T,
                                int H, int blk, cudaStream_t stream, int sms, const float* state_in) {
    const long max_items = (long)num_seqs * H * 2;
    if (max_items > (1L << 30)) return LA_ERR_UNSUPPORTED;
    tc::TileMaps m;
    const int rows = std::max(T, 1);
    if (make_tile_maps(&m, q, k, v, o, rows, H)) return LA_ERR_CUDA;
    const int chunk_tokens = ((rows + kTileRows - 1) / kTileRows) * kTileRows;  // >= every length
    const size_t aux_bytes = ((size_t)(2 * num_seqs + 2) * sizeof(int32_t) + 255) / 256 * 256;
    uint8_t* buf = nullptr;
    if (!ws_alloc(reinterpret_cast<void**>(&buf), aux_bytes, stream)) {
        return LA_ERR_ALLOC;
    }
    int* ok = reinterpret_cast<int*>(buf);
    int32_t* chunk_off = reinterpret_cast<int32_t*>(buf) + 1;
    int32_t* order = chunk_off + num_seqs + 1;
    {
        TimedLaunch tl(LA_KERNEL_AUX, stream);
        tc::varlen_prepare_kernel<<<1, 256, 0, stream>>>(cu_seqlens, num_seqs, T, chunk_tokens, ok,
                                                        chunk_off, order);
    }
    if (state_out != nullptr) {
        TimedLaunch tl(LA_KERNEL_AUX, stream);
        tc::zero_empty_states_kernel<<<dim3(num_seqs, H), 256, 0, stream>>>(state_out, cu_seqlens, ok, H,
                                                                          state_in);
    }
    tc::Params p;
    std::memset(&p, 0, sizeof(p));
    p.mode = tc::kModeVarlen;
    p.vparts = 2;
    p.blk = blk;
    p.Z = H;
    p.rows = rows;
    p.chunk_tokens = chunk_tokens;
    p.n_items = (int)max_items;
    p.cu_seqlens = cu_seqlens;
    p.chunk_off = chunk_off;
    p.seq_ok = ok;
    p.num_seqs = num_seqs;
    p.seq_order = order;
    p.state_in = state_in;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    p.state_out = state_out;
    const int grid = (int)std::min<long>(max_items, sms);
    {
        TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
        launch_main(m, p, grid, stream);
    }
    const int st = note_cuda(cudaGetLastError());
    cudaFreeAsync(buf, stream);
    return st;
}

int launch_prefill_varlen_bf16(const void* q, const void* k, const void* v, void* o,
                               float* state_out, const int32_t* cu_seqlens, int num_seqs, int T,
                               int H, int blk, cudaStream_t stream, int sms, bool three_pass,
                               int chunk_tokens, const float* state_in) {
    if (blk != 128 && blk != 64) return LA_ERR_UNSUPPORTED;
    if (chunk_tokens <= 0)
        chunk_tokens = three_pass ? choose_varlen_chunk_tokens(H, std::max(T, 1), sms)
                                  : choose_varlen_fused_chunk_tokens(H, std::max(T, 1), sms);
    chunk_tokens = ((chunk_tokens + kTileRows - 1) / kTileRows) * kTileRows;
    const long max_chunks = (long)(T + chunk_tokens - 1) / chunk_tokens + num_seqs;
    if ((long)H * max_chunks > (1L << 30)) return LA_ERR_UNSUPPORTED;
    tc::TileMaps m;
    const int rows = std::max(T, 1);
    if (make_tile_maps(&m, q, k, v, o, rows, H)) return LA_ERR_CUDA;
    const size_t aux_bytes = ((size_t)(num_seqs + 2) * sizeof(int32_t) + 255) / 256 * 256;
    const size_t ws_bytes = (size_t)H * max_chunks * kHeadDim * kHeadDim * sizeof(float);
    const size_t flag_words = three_pass ? 0 : (size_t)H * max_chunks * tc::kChainWarps + 1;  // + counter
    const size_t flag_bytes = flag_words * sizeof(int);
    uint8_t* buf = nullptr;
    if (!ws_alloc(reinterpret_cast<void**>(&buf), aux_bytes + ws_bytes + flag_bytes, stream)) {
        return LA_ERR_ALLOC;
    }
    int* ok = reinterpret_cast<int*>(buf);
    int32_t* chunk_off = reinterpret_cast<int32_t*>(buf) + 1;
    float* ws = reinterpret_cast<float*>(buf + aux_bytes);
    {
        TimedLaunch tl(LA_KERNEL_AUX, stream);
        tc::varlen_prepare_kernel<<<1, 256, 0, stream>>>(cu_seqlens, num_seqs, T, chunk_tokens, ok,
                                                        chunk_off, nullptr);
    }
    tc::Params p;
    std::memset(&p, 0, sizeof(p));
    p.mode = tc::kModeVarlen;
    p.vparts = 1;
    p.blk = blk;
    p.state_in = state_in;
    p.Z = H;
    p.rows = rows;
    p.chunk_tokens = chunk_tokens;
    p.n_items = (int)std::min<long>((long)H * max_chunks, 1L << 30);
    p.cu_seqlens = cu_seqlens;
    p.chunk_off = chunk_off;
    p.seq_ok = ok;
    p.num_seqs = num_seqs;
    p.o = reinterpret_cast<__nv_bfloat16*>(o);
    const int grid = (int)std::min<long>(p.n_items, sms);
    if (!three_pass) {
        // single pass: chunk prefixes in `ws`, flags after cu_seqlens bookkeeping
        int* chunk_flags = reinterpret_cast<int*>(buf + aux_bytes + ws_bytes);
        cudaMemsetAsync(chunk_flags, 0, flag_bytes, stream);
        if (state_out != nullptr) {
            TimedLaunch tl(LA_KERNEL_AUX, stream);
            tc::zero_empty_states_kernel<<<dim3(num_seqs, H), 256, 0, stream>>>(state_out, cu_seqlens,
                                                                              ok, H, state_in);
        }
        p.fused = 1;
        p.chain = ws;
        p.flags = chunk_flags;
        p.ticket = chunk_flags + flag_words - 1;
        p.ticket_base = g_skip_items.exchange(0);
        p.state_out = state_out;
        {
            TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
            launch_main(m, p, grid, stream);
        }
        const int st = note_cuda(cudaGetLastError());
        cudaFreeAsync(buf, stream);
        return st;
    }
    p.chunk_delta = ws;
    {
        TimedLaunch tl(LA_KERNEL_CHUNK_STATE, stream);
        tc::chunk_state_kernel<<<grid, tc::cs::kThreads, tc::cs::kSmemBytes, stream>>>(m, p);
    }
    {
        TimedLaunch tl(LA_KERNEL_CHUNK_SCAN, stream);
        dim3 sgrid(num_seqs, H);
        tc::chunk_scan_varlen_kernel<<<sgrid, 256, 0, stream>>>(ws, state_out, chunk_off, ok, H,
                                                               num_seqs, state_in);
    }
    p.prefix = ws;
    {
        TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
        launch_main(m, p, grid, stream);
    }
    const int st = note_cuda(cudaGetLastError());
    cudaFreeAsync(buf, stream);
    return st;
}

int validate_common(const void* q, const void* k, const void* v, const void* o, int d, int blk,
                    la_dtype dt) {
    if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LA_ERR_INVALID_ARG;
    if (blk < 1) return LA_ERR_INVALID_ARG;
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    if (dt == LA_BF16 && (d != 128 || (blk != 64 && blk != 128))) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

// ------------------------------------------------------------ no-alloc scratch
// Fixed scratch for la_prefill_noalloc: chunk states of the bf16 prefill for
// callers that cannot allocate device memory.  Host code must not use the
// name as a device address; it asks for the address per device below.
static __device__ __align__(256) float g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES / sizeof(float)];
float* g_noalloc_addr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device `dev`, looked up
// once per device (the first call on a device does it).
int noalloc_scratch(int dev, float** out) {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (g_noalloc_addr[dev] == nullptr) {
        void* ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return LA_ERR_CUDA;
        }
        g_noalloc_addr[dev] = static_cast<float*>(ptr);
    }
    *out = g_noalloc_addr[dev];
    return LA_OK;
}

// The bf16 chunked prefill with the chunk states in the fixed scratch.
int launch_prefill_bf16_noalloc(const void* q, const void* k, const void* v, void* o,
                                float* state_out, int BH, int N, int blk, cudaStream_t stream,
                                int dev, int sms) {
    if (blk != 128 && blk != 64) return LA_ERR_UNSUPPORTED;
    int chunk_tokens = choose_chunk_tokens(BH, N, sms);
    const int n_chunks = (N + chunk_tokens - 1) / chunk_tokens;
    const size_t ws_bytes = (size_t)BH * n_chunks * kHeadDim * kHeadDim * sizeof(float);
    if (n_chunks > 1 && ws_bytes > (size_t)LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_UNSUPPORTED;
    float* ws = nullptr;
    if (n_chunks > 1) {
        const int st = noalloc_scratch(dev, &ws);
        if (st != LA_OK) return st;
    }
    tc::TileMaps m;
    if (make_tile_maps(&m, q, k, v, o, N, BH)) return LA_ERR_CUDA;
    tc::Params p = dense_params(BH, N, chunk_tokens, o);
    p.blk = blk;
    const int grid = std::min(p.n_items, sms);
    if (n_chunks > 1) {
        launch_three_pass(m, p, ws, state_out, grid, stream);
    } else {
        p.state_out = state_out;
        TimedLaunch tl(LA_KERNEL_PREFILL_TC, stream);
        launch_main(m, p, grid, stream);
    }
    return note_cuda(cudaGetLastError());
}

}  // namespace
}  // namespace la

using namespace la;

namespace {


int decode_args_ok(const void* q, const void* k, const void* v, const void* o, int B, int H, int d,
                   la_dtype dt) {
    if (B < 1 || H < 1) return LA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LA_ERR_INVALID_ARG;
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    if ((long long)B * H > (1ll << 31) - 1) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

int slots_ok(const int32_t* slots, int num_slots, int B, int H) {
    if (slots == nullptr) return num_slots >= B ? LA_OK : LA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(slots) & 3u) != 0 || num_slots < 1) return LA_ERR_INVALID_ARG;
    if ((long long)num_slots * H > (1ll << 31) - 1) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

template <typename T>
void launch_decode(const void* q, const void* k, const void* v, float* state, void* o,
                   const int32_t* slots, int num_slots, int B, int H, int d, cudaStream_t s) {
    const T* qt = reinterpret_cast<const T*>(q);
    const T* kt = reinterpret_cast<const T*>(k);
    const T* vt = reinterpret_cast<const T*>(v);
    T* ot = reinterpret_cast<T*>(o);
    const unsigned grid = (unsigned)(B * H);
    if (d == 128)
        decode::decode_step_kernel<T, 128><<<grid, decode::kThreads, 0, s>>>(qt, kt, vt, state, ot, slots, H, num_slots);
    else
        decode::decode_step_kernel<T, 64><<<grid, decode::kThreads, 0, s>>>(qt, kt, vt, state, ot, slots, H, num_slots);
}

template <typename T, int D>
int launch_decode_q8_d(const T* q, const T* k, const T* v, int8_t* codes, float* scales, T* o,
                       const int32_t* slots, int num_slots, int B, int H, int sms, cudaStream_t s) {
    // the dynamic shared-memory size was opted into by device_setup
    auto kern = decode::decode_step_q8_kernel<T, D>;
    const int smem = decode::Q8Smem<D>::kBytes;
    const long long rows = (long long)B * H;
    int per_sm = 0;   // resident CTAs per SM (registers bound it: 2 at d = 128, 3 at d = 64)
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, decode::kThreads, smem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int grid = (int)std::min<long long>(rows, (long long)per_sm * sms);
    kern<<<grid, decode::kThreads, smem, s>>>(q, k, v, codes, scales, o, slots, H, num_slots, rows);
    return LA_OK;
}

template <typename T>
int launch_decode_q8(const void* q, const void* k, const void* v, int8_t* codes, float* scales,
                     void* o, const int32_t* slots, int num_slots, int B, int H, int d, int sms,
                     cudaStream_t s) {
    const T* qt = reinterpret_cast<const T*>(q);
    const T* kt = reinterpret_cast<const T*>(k);
    const T* vt = reinterpret_cast<const T*>(v);
    T* ot = reinterpret_cast<T*>(o);
    if (d == 128) return launch_decode_q8_d<T, 128>(qt, kt, vt, codes, scales, ot, slots, num_slots, B, H, sms, s);
    return launch_decode_q8_d<T, 64>(qt, kt, vt, codes, scales, ot, slots, num_slots, B, H, sms, s);
}

}  // namespace

extern "C" {

namespace {
int prefill_impl(const void* q, const void* k, const void* v, void* o, const float* state_in,
                 float* state_out, int B, int H, int N, int d, int blk, la_dtype dt, void* stream,
                 int chunk_tokens, int flags) {
    if (B < 1 || H < 1 || N < 1) return LA_ERR_INVALID_ARG;
    constexpr int kAllFlags = LA_FLAG_THREE_PASS | LA_FLAG_FUSED | LA_FLAG_SPLIT_V | LA_FLAG_NO_SPLIT_V;
    if ((flags & ~kAllFlags) != 0 ||
        (flags & (LA_FLAG_THREE_PASS | LA_FLAG_FUSED)) == (LA_FLAG_THREE_PASS | LA_FLAG_FUSED) ||
        (flags & (LA_FLAG_SPLIT_V | LA_FLAG_NO_SPLIT_V)) == (LA_FLAG_SPLIT_V | LA_FLAG_NO_SPLIT_V))
        return LA_ERR_INVALID_ARG;
    int st = validate_common(q, k, v, o, d, blk, dt);
    if (st != LA_OK) return st;
    if ((state_out && !aligned16(state_out)) || (state_in && !aligned16(state_in))) return LA_ERR_INVALID_ARG;
    if ((long long)B * H > (1ll << 30) || (long long)N > (1ll << 30)) return LA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int BH = B * H;
    if (dt == LA_F32) {
        const float* qf = reinterpret_cast<const float*>(q);
        const float* kf = reinterpret_cast<const float*>(k);
        const float* vf = reinterpret_cast<const float*>(v);
        float* of = reinterpret_cast<float*>(o);
        TimedLaunch tl(LA_KERNEL_PREFILL_F32, s);
        if (d == 64)
            simt::prefill_simt_kernel<64><<<BH, simt::kThreads, simt::smem_bytes<64>(), s>>>(
                qf, kf, vf, of, state_out, state_in, N, blk);
        else
            simt::prefill_simt_kernel<128><<<BH, simt::kThreads, simt::smem_bytes<128>(), s>>>(
                qf, kf, vf, of, state_out, state_in, N, blk);
        return note_cuda(cudaGetLastError());
    }
    return launch_prefill_bf16(q, k, v, o, state_out, BH, N, blk, s, sms, chunk_tokens, flags, state_in);
}
}  // namespace

int la_prefill(const void* q, const void* k, const void* v, void* o, float* state_out, int B, int H,
               int N, int d, int blk, la_dtype dt, void* stream) {
    NvtxRange nvtx_range("la_prefill");
    return la_prefill_ex(q, k, v, o, state_out, B, H, N, d, blk, dt, stream, 0, 0);
}

int la_prefill_varlen(const void* q, const void* k, const void* v, void* o, float* state_out,
                      const int32_t* cu_seqlens, int num_seqs, int total_tokens, int H, int d,
                      int blk, la_dtype dt, void* stream) {
    NvtxRange nvtx_range("la_prefill_varlen");
    return la_prefill_varlen_ex(q, k, v, o, state_out, cu_seqlens, num_seqs, total_tokens, H, d,
                                blk, dt, stream, 0, 0);
}

namespace {
int varlen_impl(const void* q, const void* k, const void* v, void* o, const float* state_in,
                float* state_out, const int32_t* cu_seqlens, int num_seqs, int total_tokens, int H,
                int d, int blk, la_dtype dt, void* stream, int chunk_tokens, int flags) {
    constexpr int kAllFlags = LA_FLAG_THREE_PASS | LA_FLAG_FUSED | LA_FLAG_SPLIT_V | LA_FLAG_NO_SPLIT_V;
    if ((flags & ~kAllFlags) != 0 ||
        (flags & (LA_FLAG_THREE_PASS | LA_FLAG_FUSED)) == (LA_FLAG_THREE_PASS | LA_FLAG_FUSED) ||
        (flags & (LA_FLAG_SPLIT_V | LA_FLAG_NO_SPLIT_V)) == (LA_FLAG_SPLIT_V | LA_FLAG_NO_SPLIT_V) ||
        ((flags & LA_FLAG_SPLIT_V) && (flags & (LA_FLAG_THREE_PASS | LA_FLAG_FUSED))) || chunk_tokens < 0)
        return LA_ERR_INVALID_ARG;
    if (num_seqs < 1 || total_tokens < 0 || H < 1 || cu_seqlens == nullptr) return LA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return LA_ERR_INVALID_ARG;
    int st = validate_common(q, k, v, o, d, blk, dt);
    if (st != LA_OK) return st;
    if ((state_out && !aligned16(state_out)) || (state_in && !aligned16(state_in))) return LA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (dt == LA_BF16 && (flags & LA_FLAG_SPLIT_V))
        return launch_prefill_varlen_split(q, k, v, o, state_out, cu_seqlens, num_seqs, total_tokens,
                                           H, blk, s, sms, state_in);
    if (dt == LA_BF16)
        return launch_prefill_varlen_bf16(q, k, v, o, state_out, cu_seqlens, num_seqs, total_tokens,
                                          H, blk, s, sms, (flags & LA_FLAG_THREE_PASS) != 0,
                                          chunk_tokens, state_in);
    int* ok = nullptr;
    if (!ws_alloc(reinterpret_cast<void**>(&ok), sizeof(int), s)) {
        return LA_ERR_ALLOC;
    }
    {
        TimedLaunch tl(LA_KERNEL_AUX, s);
        check_seqlens_kernel<<<1, 256, 0, s>>>(cu_seqlens, num_seqs, total_tokens, ok);
    }
    dim3 grid(num_seqs, H);
    const float* qf = reinterpret_cast<const float*>(q);
    const float* kf = reinterpret_cast<const float*>(k);
    const float* vf = reinterpret_cast<const float*>(v);
    float* of = reinterpret_cast<float*>(o);
    {
    TimedLaunch tl(LA_KERNEL_PREFILL_F32, s);
    if (d == 64)
        simt::prefill_simt_varlen_kernel<64><<<grid, simt::kThreads, simt::smem_bytes<64>(), s>>>(
            qf, kf, vf, of, state_out, state_in, cu_seqlens, ok, num_seqs, H, total_tokens, blk);
    else
        simt::prefill_simt_varlen_kernel<128><<<grid, simt::kThreads, simt::smem_bytes<128>(), s>>>(
            qf, kf, vf, of, state_out, state_in, cu_seqlens, ok, num_seqs, H, total_tokens, blk);
    }
    st = note_cuda(cudaGetLastError());
    cudaFreeAsync(ok, s);
    return st;
}
}  // namespace

int la_prefill_ex(const void* q, const void* k, const void* v, void* o, float* state_out, int B,
                  int H, int N, int d, int blk, la_dtype dt, void* stream, int chunk_tokens,
                  int flags) {
    NvtxRange nvtx_range("la_prefill_ex");
    return prefill_impl(q, k, v, o, nullptr, state_out, B, H, N, d, blk, dt, stream, chunk_tokens, flags);
}

int la_prefill_from_state(const void* q, const void* k, const void* v, void* o, const float* state_in,
                          float* state_out, int B, int H, int N, int d, int blk, la_dtype dt,
                          void* stream, int chunk_tokens, int flags) {
    NvtxRange nvtx_range("la_prefill_from_state");
    return prefill_impl(q, k, v, o, state_in, state_out, B, H, N, d, blk, dt, stream, chunk_tokens, flags);
}

int la_prefill_varlen_ex(const void* q, const void* k, const void* v, void* o, float* state_out,
                         const int32_t* cu_seqlens, int num_seqs, int total_tokens, int H, int d,
                         int blk, la_dtype dt, void* stream, int chunk_tokens, int flags) {
    NvtxRange nvtx_range("la_prefill_varlen_ex");
    return varlen_impl(q, k, v, o, nullptr, state_out, cu_seqlens, num_seqs, total_tokens, H, d, blk,
                       dt, stream, chunk_tokens, flags);
}

int la_prefill_varlen_from_state(const void* q, const void* k, const void* v, void* o,
                                 const float* state_in, float* state_out, const int32_t* cu_seqlens,
                                 int num_seqs, int total_tokens, int H, int d, int blk, la_dtype dt,
                                 void* stream, int chunk_tokens, int flags) {
    NvtxRange nvtx_range("la_prefill_varlen_from_state");
    return varlen_impl(q, k, v, o, state_in, state_out, cu_seqlens, num_seqs, total_tokens, H, d, blk,
                       dt, stream, chunk_tokens, flags);
}

int la_prefill_backward(const void* q, const void* k, const void* v, const void* do_, void* dq,
                        void* dk, void* dv, int B, int H, int N, int d, int blk, la_dtype dt,
                        void* stream) {
    NvtxRange nvtx_range("la_prefill_backward");
    if (B < 1 || H < 1 || N < 1 || !do_ || !dq || !dk || !dv) return LA_ERR_INVALID_ARG;
    if (!aligned16(do_) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return LA_ERR_INVALID_ARG;
    int st = validate_common(q, k, v, dq, d, blk, dt);
    if (st != LA_OK) return st;
    if ((long long)B * H > (1ll << 30) || (long long)N > (1ll << 30)) return LA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // dq_t = sum_{s <= t} (dO_t . v_s) k_s : the causal form with (q, k, v) = (dO, v, k)
    st = prefill_impl(do_, v, k, dq, nullptr, nullptr, B, H, N, d, blk, dt, stream, 0, 0);
    if (st != LA_OK) return st;
    // dk_s = sum_{t >= s} (v_s . dO_t) q_t and dv_s = sum_{t >= s} (k_s . q_t) dO_t are
    // anti-causal forms: (q, k, v) = (v, dO, q) and (k, q, dO).  The split kernel
    // runs them directly for 128-token blocks of bf16 sequences up to
    // kReverseMaxN tokens, or of any length when one CTA pair per sequence fills
    // the GPU; otherwise they are causal sums of the token-reversed sequence,
    // reversed back.
    if (dt == LA_BF16 && blk == 128 && reverse_direct_ok((long)B * H, N, sms)) {
        st = launch_prefill_reverse_bf16(v, do_, q, dk, B * H, N, s, sms);
        if (st == LA_OK) st = launch_prefill_reverse_bf16(k, q, do_, dv, B * H, N, s, sms);
        return st;
    }
    const long Z = (long)B * H;
    const size_t elems = (size_t)Z * N * d;
    const size_t esz = dt == LA_BF16 ? 2 : 4;
    const int row16 = (int)(d * esz / 16);
    uint8_t* buf = nullptr;
    if (!ws_alloc(reinterpret_cast<void**>(&buf), 5 * elems * esz, s)) {
        return LA_ERR_ALLOC;
    }
    uint8_t* rq = buf;
    uint8_t* rk = rq + elems * esz;
    uint8_t* rv = rk + elems * esz;
    uint8_t* rg = rv + elems * esz;
    uint8_t* tmp = rg + elems * esz;
    const long words = (long)elems * (long)esz / 16;
    const int grid = (int)std::min<long>((words + 255) / 256, 8L * sms);
    auto reverse = [&](const void* src, void* dst) {
        TimedLaunch tl(LA_KERNEL_AUX, s);
        reverse_tokens_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(src),
                                                   reinterpret_cast<uint4*>(dst), Z, N, row16);
    };
    reverse(q, rq);
    reverse(k, rk);
    reverse(v, rv);
    reverse(do_, rg);
    st = prefill_impl(rv, rg, rq, tmp, nullptr, nullptr, B, H, N, d, blk, dt, stream, 0, 0);
    if (st == LA_OK) {
        reverse(tmp, dk);
        st = prefill_impl(rk, rq, rg, tmp, nullptr, nullptr, B, H, N, d, blk, dt, stream, 0, 0);
    }
    if (st == LA_OK) reverse(tmp, dv);
    if (st == LA_OK) st = note_cuda(cudaGetLastError());
    cudaFreeAsync(buf, s);
    return st;
}

int la_state_increment(const void* k, const void* v, float* delta_out, int B, int H, int N, int d,
                       la_dtype dt, void* stream) {
    NvtxRange nvtx_range("la_state_increment");
    if (B < 1 || H < 1 || N < 1 || !k || !v || !delta_out) return LA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(delta_out)) return LA_ERR_INVALID_ARG;
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (dt != LA_BF16 || d != 128) return LA_ERR_UNSUPPORTED;
    if ((long long)B * H > (1ll << 30) || (long long)N > (1ll << 30)) return LA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    int st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int BH = B * H;
    // only the K and V maps are read; q and o name valid tensors of the same shape
    tc::TileMaps m;
    if (make_tile_maps(&m, k, k, v, v, N, BH)) return LA_ERR_CUDA;
    tc::Params p = dense_params(BH, N, ((N + kTileRows - 1) / kTileRows) * kTileRows, nullptr);
    p.chunk_delta = delta_out;   // one chunk per head: chunk index ws = head
    {
        TimedLaunch tl(LA_KERNEL_CHUNK_STATE, s);
        tc::chunk_state_kernel<<<std::min(p.n_items, sms), tc::cs::kThreads, tc::cs::kSmemBytes, s>>>(m, p);
    }
    return note_cuda(cudaGetLastError());
}

int la_state_prefix(const float* states, int R, int rank, float* prefix_out, int B, int H, int d,
                    void* stream) {
    NvtxRange nvtx_range("la_state_prefix");
    if (!states || !prefix_out || R < 1 || rank < 0 || rank > R || B < 1 || H < 1) return LA_ERR_INVALID_ARG;
    if (!aligned16(states) || !aligned16(prefix_out)) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    int dev = 0, sms = 0;
    int st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long n4 = (long)B * H * d * d / 4;
    {
        TimedLaunch tl(LA_KERNEL_AUX, s);
        const int grid = (int)std::min<long>((n4 + 255) / 256, 4L * sms);
        tc::state_prefix_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(states), rank, n4,
                                                     reinterpret_cast<float4*>(prefix_out));
    }
    return note_cuda(cudaGetLastError());
}

int la_decode_step(const void* q, const void* k, const void* v, float* state, void* o, int B, int H,
                   int d, la_dtype dt, void* stream) {
    NvtxRange nvtx_range("la_decode_step");
    return la_decode_step_slots(q, k, v, state, nullptr, B, o, B, H, d, dt, stream);
}

int la_decode_step_slots(const void* q, const void* k, const void* v, float* state_pool,
                         const int32_t* slots, int num_slots, void* o, int B, int H, int d,
                         la_dtype dt, void* stream) {
    NvtxRange nvtx_range("la_decode_step_slots");
    int st = decode_args_ok(q, k, v, o, B, H, d, dt);
    if (st != LA_OK) return st;
    if (!state_pool || !aligned16(state_pool)) return LA_ERR_INVALID_ARG;
    if ((st = slots_ok(slots, num_slots, B, H)) != LA_OK) return st;
    int dev = 0, sms = 0;
    if ((st = device_setup(&dev, &sms)) != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    TimedLaunch tl(LA_KERNEL_DECODE, s);
    if (dt == LA_BF16)
        launch_decode<__nv_bfloat16>(q, k, v, state_pool, o, slots, num_slots, B, H, d, s);
    else
        launch_decode<float>(q, k, v, state_pool, o, slots, num_slots, B, H, d, s);
    return note_cuda(cudaGetLastError());
}

int la_decode_step_q8(const void* q, const void* k, const void* v, int8_t* codes, float* scales,
                      const int32_t* slots, int num_slots, void* o, int B, int H, int d, la_dtype dt,
                      void* stream) {
    NvtxRange nvtx_range("la_decode_step_q8");
    int st = decode_args_ok(q, k, v, o, B, H, d, dt);
    if (st != LA_OK) return st;
    if (!codes || !scales || !aligned16(codes) || !aligned16(scales)) return LA_ERR_INVALID_ARG;
    if ((st = slots_ok(slots, num_slots, B, H)) != LA_OK) return st;
    int dev = 0, sms = 0;
    if ((st = device_setup(&dev, &sms)) != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    TimedLaunch tl(LA_KERNEL_DECODE, s);
    st = dt == LA_BF16
             ? launch_decode_q8<__nv_bfloat16>(q, k, v, codes, scales, o, slots, num_slots, B, H, d, sms, s)
             : launch_decode_q8<float>(q, k, v, codes, scales, o, slots, num_slots, B, H, d, sms, s);
    if (st != LA_OK) return st;
    return note_cuda(cudaGetLastError());
}

int la_state_quantize_q8(const float* state, int8_t* codes, float* scales, long long n_heads, int d,
                         void* stream) {
    NvtxRange nvtx_range("la_state_quantize_q8");
    if (n_heads < 1 || !state || !codes || !scales) return LA_ERR_INVALID_ARG;
    if (!aligned16(state) || !aligned16(codes) || !aligned16(scales)) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    int dev = 0, sms = 0;
    int st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long rows = n_heads * d;
    const long long warps_needed = (rows * (d / 4) + 31) / 32;
    const int grid = (int)std::min<long long>((warps_needed + 7) / 8, 8LL * sms);
    TimedLaunch tl(LA_KERNEL_AUX, s);
    if (d == 128)
        decode::state_quantize_q8_kernel<128><<<grid, 256, 0, s>>>(state, codes, scales, rows);
    else
        decode::state_quantize_q8_kernel<64><<<grid, 256, 0, s>>>(state, codes, scales, rows);
    return note_cuda(cudaGetLastError());
}

int la_state_dequantize_q8(const int8_t* codes, const float* scales, float* state, long long n_heads,
                           int d, void* stream) {
    NvtxRange nvtx_range("la_state_dequantize_q8");
    if (n_heads < 1 || !state || !codes || !scales) return LA_ERR_INVALID_ARG;
    if (!aligned16(state) || !aligned16(codes) || !aligned16(scales)) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    int dev = 0, sms = 0;
    int st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long n4 = n_heads * d * d / 4;
    const int grid = (int)std::min<long long>((n4 + 255) / 256, 8LL * sms);
    TimedLaunch tl(LA_KERNEL_AUX, s);
    if (d == 128)
        decode::state_dequantize_q8_kernel<128><<<grid, 256, 0, s>>>(codes, scales, state, n4);
    else
        decode::state_dequantize_q8_kernel<64><<<grid, 256, 0, s>>>(codes, scales, state, n4);
    return note_cuda(cudaGetLastError());
}

const char* la_status_string(int status) {
    switch (status) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
        case LA_ERR_CUDA: return "LA_ERR_CUDA";
        case LA_ERR_ALLOC: return "LA_ERR_ALLOC";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
        case LA_ERR_BAD_SEQLENS: return "LA_ERR_BAD_SEQLENS";
        case LA_ERR_BAD_SLOT: return "LA_ERR_BAD_SLOT";
        default: return "LA_UNKNOWN_STATUS";
    }
}

int la_get_last_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    int dev_status = LA_OK;
    if (cudaMemcpyFromSymbol(&dev_status, la::g_device_status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    const int zero = LA_OK;
    cudaMemcpyToSymbol(la::g_device_status, &zero, sizeof(int));
    int host_status;
    {
        std::lock_guard<std::mutex> lk(g_mutex);
        host_status = g_host_status;
        g_host_status = LA_OK;
    }
    if (dev_status != LA_OK) return dev_status;
    return host_status;
}

int la_device_sm_count(void) {
    int dev = 0, sms = 0;
    if (device_setup(&dev, &sms) != LA_OK) return 0;
    return sms;
}

int la_prefill_noalloc(const void* q, const void* k, const void* v, void* o, float* state_out,
                       int B, int H, int N, int d, int blk, la_dtype dt, void* stream) {
    NvtxRange nvtx_range("la_prefill_noalloc");
    if (B < 1 || H < 1 || N < 1) return LA_ERR_INVALID_ARG;
    int st = validate_common(q, k, v, o, d, blk, dt);
    if (st != LA_OK) return st;
    if (dt != LA_BF16) return LA_ERR_UNSUPPORTED;
    if (state_out && !aligned16(state_out)) return LA_ERR_INVALID_ARG;
    if ((long long)B * H > (1ll << 30) || (long long)N > (1ll << 30)) return LA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    return launch_prefill_bf16_noalloc(q, k, v, o, state_out, B * H, N, blk,
                                       reinterpret_cast<cudaStream_t>(stream), dev, sms);
}

int la_timing_enable(int max_launches) {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_timing.ev.empty()) cudaDeviceSynchronize();
    timing_release();
    if (max_launches <= 0) return LA_OK;
    g_timing.ev.resize(2 * (size_t)max_launches);
    g_timing.kid.assign(max_launches, -1);
    for (auto& e : g_timing.ev) {
        if (cudaEventCreate(&e) != cudaSuccess) {
            cudaGetLastError();
            e = nullptr;
            timing_release();
            return LA_ERR_CUDA;
        }
    }
    g_timing.cap = max_launches;
    g_timing.enabled = true;
    return LA_OK;
}

int la_timing_read(int kernel_id, double* total_ms, int* launches) {
    if (kernel_id < 0 || kernel_id >= LA_NUM_KERNEL_IDS || !total_ms || !launches)
        return LA_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_mutex);
    double sum = 0.0;
    for (int i = 0; i < g_timing.used; ++i) {
        if (g_timing.kid[i] != kernel_id) continue;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_timing.ev[2 * i], g_timing.ev[2 * i + 1]) != cudaSuccess) {
            cudaGetLastError();
            return LA_ERR_CUDA;
        }
        sum += ms;
    }
    *total_ms = sum;
    *launches = g_timing.launches[kernel_id];
    return LA_OK;
}

const char* la_prefill_main_kernel(void) { return g_main_kernel.load(); }

int la_set_wait_limit_ns(unsigned long long limit_ns, unsigned long long* previous_ns) {
    int dev = 0, sms = 0;
    int st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    const unsigned long long v = limit_ns == 0 ? kDefaultWaitLimitNs : limit_ns;
    if (previous_ns != nullptr &&
        cudaMemcpyFromSymbol(previous_ns, la::g_wait_limit_ns, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (cudaMemcpyToSymbol(la::g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return LA_OK;
}

int la_debug_skip_lookback_items(int count) {
    if (count < 0) return LA_ERR_INVALID_ARG;
    g_skip_items.store(count);
    return LA_OK;
}

int la_debug_stall_split_load(int tile) {
    if (tile < -1) return LA_ERR_INVALID_ARG;
    g_stall_tile.store(tile + 1);
    return LA_OK;
}

int la_debug_occupy_sms(int ctas, unsigned long long duration_ns, void* stream) {
    if (ctas < 1 || duration_ns > 1000000000ull) return LA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    int st = device_setup(&dev, &sms);
    if (st != LA_OK) return st;
    if (cudaFuncSetAttribute(occupy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOccupySmem) !=
        cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    occupy_kernel<<<ctas, 32, kOccupySmem, reinterpret_cast<cudaStream_t>(stream)>>>(duration_ns);
    return note_cuda(cudaGetLastError());
}

int la_debug_fail_allocations(int count) {
    if (count < 0) return LA_ERR_INVALID_ARG;
    g_fail_allocs.store(count);
    return LA_OK;
}

int la_binary_version(void) {
    int dev = 0, sms = 0;
    if (device_setup(&dev, &sms) != LA_OK) return LA_ERR_CUDA;
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, tc::prefill_seq_kernel<false>) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return a.binaryVersion;
}

const char* la_kernel_name(int kernel_id) {
    switch (kernel_id) {
        case LA_KERNEL_PREFILL_TC: return "prefill_main";
        case LA_KERNEL_CHUNK_STATE: return "chunk_state_kernel";
        case LA_KERNEL_CHUNK_SCAN: return "chunk_scan_kernel";
        case LA_KERNEL_PREFILL_F32: return "prefill_simt_kernel";
        case LA_KERNEL_DECODE: return "decode_step_kernel";
        case LA_KERNEL_AUX: return "check_seqlens_kernel";
        default: return "unknown";
    }
}

}  // extern "C"
