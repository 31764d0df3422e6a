/*
 * lightning.h -- C ABI of liblightning.so: causal linear attention
 * ("Lightning Attention") on NVIDIA B200 (sm_100a).  Entry points: prefill
 * (dense and packed variable-length, optionally continued from a given
 * state), its backward, the state increment and prefix used for sequence
 * parallelism, and decode (fp32 state, a slot pool with padding rows, and an
 * 8-bit state with its conversions); status and timing queries.
 *
 * The operation (no softmax, no scale, no normaliser, diagonal included):
 *
 *     S_t = sum_{s <= t} k_s^T v_s          (d x d state, row = key dim)
 *     o_t = q_t S_t = sum_{s <= t} (q_t . k_s) v_s
 *
 * computed block-wise: inside a block of `blk` tokens with the masked left
 * product (Q K^T ⊙ M) V, across blocks with the right product Q (K^T V) from
 * the running state, so no cumulative sum over tokens is formed.  Sources:
 * section 1 of "MiniMax-01技術報告解讀以及與DeepSeek-V3對比" (m.futurefh.com:
 * intra-block left product, inter-block right product, no slow cumsum);
 * "The Core Tech: Lightning Attention" of "MiniMax M2.1" (nabfollower.com:
 * associativity (QK^T)V = Q(K^T V)); section 3 of the futurefh page (prefill and
 * decode run separately); section 4 (packed sequences).
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Every pointer is a DEVICE pointer owned by the caller; the library never
 *    frees or retains it.  Tensors are dense, contiguous, row-major.
 *  - q, k, v, o have element type `dt` (fp32 or bf16); states are always fp32.
 *  - Pointers must be 16-byte aligned (LA_ERR_INVALID_ARG otherwise).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    All work is enqueued asynchronously on it; the call returns after
 *    launching.  Argument errors are returned synchronously and nothing is
 *    launched.  Errors detected on the device (malformed cu_seqlens, a bounded
 *    wait that gave up) are recorded in a device status word that
 *    la_get_last_error() reports.  The library never aborts, prints or traps.
 *  - Supported sizes: d in {64, 128}; the bf16 tensor-core path needs d == 128
 *    and blk in {64, 128}; the fp32 path accepts any blk >= 1 with d in {64, 128}.
 *    N may be any value >= 1 (need not be a multiple of blk).
 *  - Scratch: long sequences are split into chunks processed in parallel; the
 *    per-chunk states live in a workspace the library takes from the stream-
 *    ordered allocator (cudaMallocAsync / cudaFreeAsync on `stream`).
 *  - Thread safety: calls from several threads, on different streams, may run
 *    concurrently.  The device status word (la_get_last_error) and the
 *    bounded-wait limit (la_set_wait_limit_ns) are per device, shared by all
 *    streams and threads of the process.
 */
#ifndef LIGHTNING_H_
#define LIGHTNING_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, non-positive size  */
    LA_ERR_UNSUPPORTED = -2,   /* valid but unsupported (d, blk, dtype) combo */
    LA_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed           */
    LA_ERR_ALLOC = -4,         /* workspace allocation failed                 */
    LA_ERR_TIMEOUT = -5,       /* a bounded device-side wait gave up          */
    LA_ERR_BAD_SEQLENS = -6,   /* cu_seqlens not 0..total_tokens non-decreasing */
    LA_ERR_BAD_SLOT = -7       /* a decode slot id >= num_slots (row skipped)  */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/*
 * la_prefill -- causal linear attention over B*H independent sequences.
 *   q, k, v  : [B, H, N, d] of dt (read only)
 *   o        : [B, H, N, d] of dt (written)
 *   state_out: [B, H, d, d] fp32, final state S_{N-1} = K^T V (written; may be
 *              NULL when the caller does not need it)
 *   blk      : block size of the intra/inter split (section 1 of the futurefh
 *              page).  The result is mathematically independent of blk; blk
 *              changes only the rounding path.
 * Returns LA_OK or an la_status error.
 */
int la_prefill(const void* q, const void* k, const void* v, void* o, float* state_out,
               int B, int H, int N, int d, int blk, la_dtype dt, void* stream);

/*
 * la_prefill_ex -- la_prefill with explicit scheduling controls.
 *   chunk_tokens: length of the sequence chunks processed in parallel (a
 *                 multiple of 128 on the bf16 path); 0 = library heuristic;
 *                 a value >= N forces one chunk per sequence.
 *   flags       : LA_FLAG_* bits below; 0 = default schedule.
 */
#define LA_FLAG_THREE_PASS 1   /* chunk states, scan, then outputs (3 launches) */
#define LA_FLAG_FUSED      2   /* single persistent launch with look-back (the
                                  default): each chunk publishes its inclusive
                                  state prefix for the next one              */
#define LA_FLAG_SPLIT_V    4   /* split the value columns of every head over two
                                  CTAs (independent halves of S and O); with
                                  blk 64 only where each sequence is one chunk
                                  (otherwise whole rows are kept)             */
#define LA_FLAG_NO_SPLIT_V 8   /* never split the value columns               */
int la_prefill_ex(const void* q, const void* k, const void* v, void* o, float* state_out,
                  int B, int H, int N, int d, int blk, la_dtype dt, void* stream,
                  int chunk_tokens, int flags);

/*
 * la_prefill_varlen -- packed variable-length prefill (data packing, section 4
 * of the futurefh page).  Sequence j occupies tokens [cu_seqlens[j],
 * cu_seqlens[j+1]) of every head; the state restarts at zero at each sequence
 * start.
 *   q, k, v, o : [H, total_tokens, d] of dt, head-major packed
 *   cu_seqlens : [num_seqs + 1] int32 DEVICE array, cu_seqlens[0] == 0,
 *                non-decreasing, cu_seqlens[num_seqs] == total_tokens.  It is
 *                checked on the device; a malformed array sets
 *                LA_ERR_BAD_SEQLENS in the device status and no output is
 *                written.  Empty sequences are allowed (zero state).
 *   state_out  : [num_seqs, H, d, d] fp32 final state per sequence (may be NULL)
 */
int la_prefill_varlen(const void* q, const void* k, const void* v, void* o, float* state_out,
                      const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                      int H, int d, int blk, la_dtype dt, void* stream);

/*
 * la_prefill_varlen_ex -- la_prefill_varlen with scheduling controls.
 *   chunk_tokens: chunk length of the chunked schedules, a multiple of 128,
 *                 0 = library choice (ignored by LA_FLAG_SPLIT_V).
 *   flags: 0 = default; LA_FLAG_THREE_PASS or LA_FLAG_FUSED pick a chunked
 *          schedule over whole value rows (optionally with LA_FLAG_NO_SPLIT_V);
 *          LA_FLAG_SPLIT_V (alone; bf16, blk 128 or 64) runs every (sequence, head)
 *          unchunked with its value columns split over two CTAs, longest
 *          sequences first.  Other combinations return LA_ERR_INVALID_ARG.
 */
int la_prefill_varlen_ex(const void* q, const void* k, const void* v, void* o, float* state_out,
                         const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                         int H, int d, int blk, la_dtype dt, void* stream,
                         int chunk_tokens, int flags);

/*
 * la_prefill_from_state / la_prefill_varlen_from_state -- the prefills above
 * continued from a given state: S_{-1} = state_in instead of zero, so
 *     o_t = q_t (state_in + sum_{s <= t} k_s^T v_s),  state_out = state_in + K^T V.
 * A sequence processed in pieces (chunked prefill, a prompt extended after
 * decoding) gives the same result as in one call: prefill(A) then
 * prefill_from_state(B, state_out of A) equals prefill(A ++ B) on B.
 *   state_in : dense [B, H, d, d] / packed [num_seqs, H, d, d] fp32, the
 *              layout of state_out (read only; NULL = zero start, which is
 *              la_prefill_ex / la_prefill_varlen_ex).  It may be the same
 *              array as state_out (each head's state is read before its final
 *              state is written).  An empty packed sequence gets
 *              state_out = state_in.
 * Every other argument, the flags and the errors are those of la_prefill_ex /
 * la_prefill_varlen_ex.  The starting state of the block-wise form (section 1
 * of the futurefh page) is the running state; the pages do not name this
 * entry point.
 */
int la_prefill_from_state(const void* q, const void* k, const void* v, void* o, const float* state_in,
                          float* state_out, int B, int H, int N, int d, int blk, la_dtype dt,
                          void* stream, int chunk_tokens, int flags);
int la_prefill_varlen_from_state(const void* q, const void* k, const void* v, void* o,
                                 const float* state_in, float* state_out, const int32_t* cu_seqlens,
                                 int num_seqs, int total_tokens, int H, int d, int blk, la_dtype dt,
                                 void* stream, int chunk_tokens, int flags);

/*
 * la_prefill_backward -- gradients of L = sum_t dO_t . o_t for o = la_prefill
 * (q, k, v) (zero starting state), the training direction:
 *     dq_t = sum_{s <= t} (dO_t . v_s) k_s     (the causal form of (dO, v, k))
 *     dk_s = sum_{t >= s} (dO_t . v_s) q_t     (the anti-causal form of (v, dO, q))
 *     dv_s = sum_{t >= s} (q_t . k_s) dO_t     (the anti-causal form of (k, q, dO))
 *   q, k, v, do_ : [B, H, N, d] of dt (read only); dq, dk, dv : [B, H, N, d]
 *   of dt (written).  Same dtype, d, blk rules as la_prefill.  For bf16 with
 *   blk = 128 the anti-causal forms run directly (the tiles of each sequence
 *   taken from the last) and no scratch is used when N <= 16384, or for any N
 *   when 2*B*H is between 80 % and 100 % of the SM count (one CTA pair per
 *   sequence fills the GPU); otherwise they are causal forms of the
 *   token-reversed sequence, reversed back, with five tensors of the input
 *   size of scratch from the stream-ordered allocator (LA_ERR_ALLOC if that
 *   fails).  The pages
 *   give no backward pass (training is the context of section 2 of the
 *   futurefh page); this is the derivative of the forward definition.
 */
int la_prefill_backward(const void* q, const void* k, const void* v, const void* do_, void* dq,
                        void* dk, void* dv, int B, int H, int N, int d, int blk, la_dtype dt,
                        void* stream);

/*
 * Sequence parallelism across GPUs (the improved linear-attention sequence
 * parallelism, LASP, that section 2 of the futurefh page names for unbounded
 * context windows; the pages give no algorithm, this is its plain reading).  A sequence split over R ranks, rank r
 * holding tokens [r N/R, (r+1) N/R) of every (batch, head), is prefilled as
 *   1. la_state_increment: dS_r = K_r^T V_r of the rank's tokens;
 *   2. all-gather of dS over the ranks (the caller's collective, e.g. NCCL);
 *   3. la_state_prefix: S_in,r = sum_{r' < r} dS_r';
 *   4. la_prefill_from_state on the rank's tokens from S_in,r.
 * The last rank's state_out is the whole sequence's final state.
 *
 * la_state_increment -- delta_out[B,H,d,d] (fp32, written) = K^T V over the
 *   N tokens of k, v [B,H,N,d] (read only).  bf16 with d = 128 only
 *   (LA_ERR_UNSUPPORTED otherwise).
 * la_state_prefix -- prefix_out[B,H,d,d] = sum_{r < rank} states[r] (zero for
 *   rank 0), summed in rank order; states is [R][B,H,d,d] fp32 (read only),
 *   0 <= rank <= R, d in {64, 128}.
 */
int la_state_increment(const void* k, const void* v, float* delta_out, int B, int H, int N, int d,
                       la_dtype dt, void* stream);
int la_state_prefix(const float* states, int R, int rank, float* prefix_out, int B, int H, int d,
                    void* stream);

/*
 * la_decode_step -- one token per sequence (prefill and decode are separate,
 * section 3 of the futurefh page):  S <- S + k^T v ;  o = q S  (the update
 * includes the current token, so prefill(N) + step == prefill(N+1)).
 *   q, k, v : [B, H, d] of dt (read only)
 *   state   : [B, H, d, d] fp32, read and updated in place
 *   o       : [B, H, d] of dt (written)
 */
int la_decode_step(const void* q, const void* k, const void* v, float* state, void* o,
                   int B, int H, int d, la_dtype dt, void* stream);

/*
 * la_decode_step_slots -- batched decode over a pool of states.  Section 3 of
 * the futurefh page pads batches in several levels to keep padding overhead
 * small; here row b of a batch padded to B rows addresses the state
 * state_pool[slots[b]], and a row with a negative slot is padding: its o row
 * is written as zeros and no state is read or written.  So a batch padded up
 * to a fixed level (for one captured CUDA graph per level) costs state
 * traffic only for its live rows.
 *   q, k, v  : [B, H, d] of dt (read only);  o : [B, H, d] of dt (written)
 *   state_pool: [num_slots, H, d, d] fp32, live slots updated in place
 *   slots    : [B] int32 on the device; NULL means row b uses slot b (then
 *              num_slots >= B).  Each live slot may appear once per call
 *              (a repeated slot gives an unspecified result for that slot, but
 *              no access outside the pool).
 * A slot >= num_slots is recorded as LA_ERR_BAD_SLOT in the device status and
 * its row is treated as padding.
 */
int la_decode_step_slots(const void* q, const void* k, const void* v, float* state_pool,
                         const int32_t* slots, int num_slots, void* o, int B, int H, int d,
                         la_dtype dt, void* stream);

/*
 * 8-bit decode state.  The yuliangy.com digest of the MiniMax-01 report
 * credits 8-bit quantisation with fitting more than a million tokens on one
 * eight-GPU machine; the format is this library's reading: row i of a head's
 * state (key dimension i) is int8 codes c_ij in [-127, 127] plus one fp32
 * scale a_i, S_ij = c_ij * a_i.  Quantising a row: m = max_j |x_j|; if
 * m < 2^-100 the row is stored as zero (a = 0); else a = m / 127 and
 * c_j = nearest-even integer to x_j * (127 / m), each one correctly rounded
 * fp32 operation, so results are reproducible bit for bit.
 *   codes : [n_heads, d, d] int8;  scales : [n_heads, d] fp32 (16-byte aligned)
 *
 * la_state_quantize_q8   fp32 states [n_heads, d, d] -> (codes, scales)
 * la_state_dequantize_q8 (codes, scales) -> fp32 states (one fp32 product each)
 *
 * la_decode_step_q8 -- la_decode_step_slots on the 8-bit state:
 *     s_ij = fma(k_i, v_j, c_ij * a_i)   (fp32, rounded once)
 *     o_j  = sum_i q_i s_ij               (fp32 accumulation)
 *     codes, scales <- the rows of s quantised as above
 *   codes : [num_slots, H, d, d] int8, scales : [num_slots, H, d] fp32, in place
 *   slots, padding rows and LA_ERR_BAD_SLOT as for la_decode_step_slots.
 * State traffic per head-step is 2 (d*d + 4 d) bytes against 8 d*d for fp32.
 */
int la_state_quantize_q8(const float* state, int8_t* codes, float* scales, long long n_heads, int d,
                         void* stream);
int la_state_dequantize_q8(const int8_t* codes, const float* scales, float* state, long long n_heads,
                           int d, void* stream);
int la_decode_step_q8(const void* q, const void* k, const void* v, int8_t* codes, float* scales,
                      const int32_t* slots, int num_slots, void* o, int B, int H, int d, la_dtype dt,
                      void* stream);

/* Human-readable name of an la_status value (static storage). */
const char* la_status_string(int status);

/*
 * la_get_last_error -- sticky error: the first device-side error recorded
 * since the last call (see la_status), else the last asynchronous CUDA error,
 * else LA_OK.  It synchronises the current device and clears the status.
 * The status word is one per device for the whole process, not one per
 * stream: an error recorded by work on any stream or thread is reported to,
 * and cleared by, whichever caller asks first.  Entry points may be called
 * from several threads and streams at once; callers that need to attribute
 * a device error to one stream must serialise their checks.
 */
int la_get_last_error(void);

/* Number of SMs the library schedules for on the current device (0 on error). */
int la_device_sm_count(void);

/*
 * Per-kernel timing (instrumentation).  While enabled, every kernel launch the
 * library makes on the current device is bracketed by a pair of CUDA events
 * recorded on the launch's own stream, into a pool of `max_launches` pairs
 * (launches beyond the pool are counted but not timed).  Kernel ids:
 *   LA_KERNEL_PREFILL_TC  main tensor-core prefill pass (outputs), whichever
 *                         kernel variant la_prefill_main_kernel() names
 *   LA_KERNEL_CHUNK_STATE per-chunk K^T V (first pass of the chunk scan)
 *   LA_KERNEL_CHUNK_SCAN  exclusive prefix over chunk states
 *   LA_KERNEL_PREFILL_F32 fp32 CUDA-core prefill (dense and varlen)
 *   LA_KERNEL_DECODE      decode step
 *   LA_KERNEL_AUX         small helper kernels (cu_seqlens check, ...)
 * la_timing_enable(n) starts a new measurement with room for n launches
 * (n <= 0 disables timing and releases the events).  la_timing_read
 * synchronises the device and returns the summed event time in milliseconds
 * and the launch count of one kernel id since la_timing_enable.
 */
#define LA_KERNEL_PREFILL_TC 0
#define LA_KERNEL_CHUNK_STATE 1
#define LA_KERNEL_CHUNK_SCAN 2
#define LA_KERNEL_PREFILL_F32 3
#define LA_KERNEL_DECODE 4
#define LA_KERNEL_AUX 5
#define LA_NUM_KERNEL_IDS 6
int la_timing_enable(int max_launches);
int la_timing_read(int kernel_id, double* total_ms, int* launches);
const char* la_kernel_name(int kernel_id);

/*
 * Name of the kernel the most recent bf16 prefill call (from any thread)
 * launched for its output pass: "prefill_tc_kernel<128>" (whole value rows,
 * chain warps), "prefill_tc_kernel<64>" (value columns split over two CTAs,
 * single pass with look-back), "prefill_tc_kernel<128,64>" (64-token blocks,
 * whole value rows), "prefill_seq_kernel" (value columns split, no look-back)
 * or "prefill_seq64_kernel" (the same with 64-token blocks); "" before the
 * first call.  Informational: a static string, never freed.
 */
const char* la_prefill_main_kernel(void);

/*
 * Bounded waits.  Every wait of the device code (an mbarrier phase, a chunk
 * prefix published by another CTA, a bulk copy landing) gives up after a time
 * limit of %globaltimer: the kernel then records LA_ERR_TIMEOUT in the device
 * status, every role of the CTA leaves its loop, the copies and MMAs already
 * issued are let land, TMEM is freed and the kernel returns; the outputs of
 * that call are unspecified, the context stays usable.
 * la_set_wait_limit_ns -- set that limit on the current device for kernels
 *   launched after the call returns (0 restores the default of 2 s); the old
 *   value is stored in *previous_ns when previous_ns is not NULL.  One value
 *   per device for the whole process.  Synchronous; not for use during
 *   stream capture.
 */
int la_set_wait_limit_ns(unsigned long long limit_ns, unsigned long long* previous_ns);

/*
 * la_debug_fail_allocations -- host-side failure injection for tests: the next
 * `count` workspace allocations of the library (from any thread) fail as if
 * the stream-ordered allocator were out of memory, so the calls that need
 * them return LA_ERR_ALLOC before launching anything; 0 cancels.  Nothing
 * runs on the device.  Returns LA_OK (LA_ERR_INVALID_ARG if count < 0).
 */
int la_debug_fail_allocations(int count);

/*
 * Test hooks for the failure paths of the look-back (single pass) schedule.
 * la_debug_skip_lookback_items -- the next look-back launch on any stream
 *   starts its work-item tickets at `count` instead of 0: the first `count`
 *   items are never processed, so the chunks that follow them wait for a
 *   state prefix that is never published, and their bounded waits run out
 *   (LA_ERR_TIMEOUT in the device status).  One launch only; 0 cancels.
 * la_debug_occupy_sms -- launch `ctas` CTAs on `stream`, each holding most of
 *   an SM's shared memory and waiting `duration_ns` (at most 1 s) on the
 *   clock before it exits: other kernels then run on the remaining SMs.
 * Both return LA_OK or LA_ERR_INVALID_ARG / LA_ERR_CUDA.  They exist for
 * tests; nothing else calls them.
 */
int la_debug_skip_lookback_items(int count);
int la_debug_occupy_sms(int ctas, unsigned long long duration_ns, void* stream);

/*
 * la_debug_stall_split_load -- the next launch of a split-value-column kernel
 * (prefill_seq_kernel, prefill_seq64_kernel) leaves the loads of the `tile`-th
 * tile each CTA processes (counted from 0) unissued: the MMA issuers' bounded
 * waits for it run out, LA_ERR_TIMEOUT is recorded, and every role leaves after
 * letting its own loads and MMAs complete.  One launch only; -1 cancels.
 * Returns LA_OK or LA_ERR_INVALID_ARG.  A test hook; nothing else calls it.
 */
int la_debug_stall_split_load(int tile);

/*
 * la_binary_version -- the compute capability the library's kernels were
 * compiled for, as major * 10 + minor (100 for sm_100a), read from the
 * loaded code object on the current device; LA_ERR_CUDA if it cannot be read.
 */
int la_binary_version(void);

/*
 * la_prefill_noalloc -- la_prefill (bf16, d = 128) that allocates no device
 * memory.  The paper has no counterpart to this entry point: it is a
 * packaging variant of the bf16 prefill for callers that cannot call
 * cudaMalloc or the stream-ordered allocator, for example code running inside
 * a framework that has already reserved nearly all device memory for its own
 * pool (so any allocation by a library would fail), or a runtime that forbids
 * allocations outside its planned arena.
 *
 * Arguments, layouts, results and errors are those of la_prefill.  The
 * per-chunk states that la_prefill keeps in an allocated workspace live here
 * in one fixed array inside the library, LA_NOALLOC_SCRATCH_BYTES large,
 * which every GPU that loads the library holds until the process exits.  It
 * always runs the three-pass schedule over whole value rows, with the chunk
 * length la_prefill_ex chooses for flags LA_FLAG_THREE_PASS |
 * LA_FLAG_NO_SPLIT_V and chunk_tokens = 0 (which depends on B*H, N and the
 * SM count, and is never shorter than 512 tokens).  With n_chunks =
 * ceil(N / chunk length), the chunk states take B*H*n_chunks*d*d*4 bytes; if
 * that exceeds the array the call returns LA_ERR_UNSUPPORTED and launches
 * nothing.  B*H*ceil(N/512) <= 256 always fits.  (A sequence that fits one
 * chunk needs no scratch at all.)
 *
 * The first call on each device looks up the device address of the array
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls on a device share the one array and
 * it keeps whatever the last call left in it (every entry is overwritten
 * before it is read, so nothing needs clearing); two calls whose work
 * overlaps on the GPU (different streams, no ordering between them) race on
 * it and must not be issued.
 */
#define LA_NOALLOC_SCRATCH_BYTES (16u << 20)
int la_prefill_noalloc(const void* q, const void* k, const void* v, void* o, float* state_out,
                       int B, int H, int N, int d, int blk, la_dtype dt, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_H_ */
