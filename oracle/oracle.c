/*
 * oracle.c -- plain, slow, fp64 CPU reference for causal linear attention
 * ("Lightning Attention").
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may include, link, load or call this file.  Only the
 * tests, the smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or helper with the CUDA kernels.
 *
 * What is computed (all forms are the same mathematical object):
 *
 *     o_t = sum_{s <= t} (q_t . k_s) v_s            (causal, diagonal included,
 *                                                    no softmax, no scale,
 *                                                    no normaliser)
 *     S_t = sum_{s <= t} k_s^T v_s                   (d x d running state,
 *                                                    row = key dim, col = value dim)
 *     o_t = q_t S_t
 *
 * Sources (web pages about the MiniMax-01 report):
 *  - "MiniMax-01技術報告解讀以及與DeepSeek-V3對比" (m.futurefh.com), section 1
 *    ("core innovation: linear attention"): lightning attention splits the
 *    attention computation into an intra-block part computed with the left
 *    product and an inter-block part computed with the right product, which
 *    avoids the slow cumulative sum.
 *  - "MiniMax M2.1 (the 'linear' revolution)" (nabfollower.com), section
 *    "The Core Tech: Lightning Attention": by associativity of matrix products
 *    (Q K^T) V is regrouped as Q (K^T V), bringing the cost from O(N^2 d) to
 *    O(N d^2); the closing analogy of the same page: linear attention keeps a
 *    fixed-size summary (hidden state) while it scans the sequence.
 *  - Section 3 of the first page ("efficient inference framework"): prefill and
 *    decode are executed separately.  Section 4 ("long-context training"):
 *    sequences are packed (data packing), which the varlen form models.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 * no decay, no feature map, no 1/sqrt(d) scale, no normalising denominator;
 * the diagonal s == t is included; the state used for block i excludes block
 * i; a decode step updates the state with the new token before reading it.
 *
 * Layouts: q, k, v, o are [BH][N][d] row-major (BH = batch*heads flattened);
 * states are [BH][d][d] row-major with row index = key dim.  Varlen inputs are
 * packed [H][T][d]; cu_seqlens has num_seqs+1 entries; states are
 * [num_seqs][H][d][d].
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Quadratic masked form, straight from the definition (the "left product"
 * (Q K^T ⊙ M) V of section 1 of the futurefh page, applied to the whole
 * sequence with M lower-triangular including the diagonal).  O(N^2 d).
 */
void oracle_prefill_quadratic(const double* q, const double* k, const double* v,
                              double* o, long BH, long N, long d) {
    long bh;
#pragma omp parallel for schedule(dynamic)
    for (bh = 0; bh < BH; ++bh) {
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        double* O = o + bh * N * d;
        for (long t = 0; t < N; ++t) {
            for (long j = 0; j < d; ++j) O[t * d + j] = 0.0;
            for (long s = 0; s <= t; ++s) {
                double score = 0.0;
                for (long c = 0; c < d; ++c) score += Q[t * d + c] * K[s * d + c];
                for (long j = 0; j < d; ++j) O[t * d + j] += score * V[s * d + j];
            }
        }
    }
}

/*
 * Recurrent (scan) form: the fixed-size state of the nabfollower page's
 * analogy.  For t = 0..N-1:  S <- S + k_t^T v_t ;  o_t = q_t S.
 * state_in may be NULL (S starts at zero); state_out may be NULL.  O(N d^2).
 */
void oracle_prefill_recurrent(const double* q, const double* k, const double* v,
                              const double* state_in, double* o, double* state_out,
                              long BH, long N, long d) {
    long bh;
#pragma omp parallel for schedule(dynamic)
    for (bh = 0; bh < BH; ++bh) {
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        double* O = o + bh * N * d;
        double* S = (double*)malloc((size_t)(d * d) * sizeof(double));
        if (state_in)
            memcpy(S, state_in + bh * d * d, (size_t)(d * d) * sizeof(double));
        else
            memset(S, 0, (size_t)(d * d) * sizeof(double));
        for (long t = 0; t < N; ++t) {
            for (long i = 0; i < d; ++i)
                for (long j = 0; j < d; ++j) S[i * d + j] += K[t * d + i] * V[t * d + j];
            for (long j = 0; j < d; ++j) {
                double acc = 0.0;
                for (long i = 0; i < d; ++i) acc += Q[t * d + i] * S[i * d + j];
                O[t * d + j] = acc;
            }
        }
        if (state_out) memcpy(state_out + bh * d * d, S, (size_t)(d * d) * sizeof(double));
        free(S);
    }
}

/*
 * Gradients of L = sum_t dO_t . o_t with respect to q, k, v, from the
 * quadratic definition o_t = sum_{s <= t} (q_t . k_s) v_s differentiated term
 * by term (the pages give no backward pass; training is the context of the
 * LASP+ passage of the futurefh page, section 2):
 *     dq_t = sum_{s <= t} (dO_t . v_s) k_s
 *     dk_s = sum_{t >= s} (dO_t . v_s) q_t
 *     dv_s = sum_{t >= s} (q_t . k_s) dO_t
 * O(N^2 d).  Layout as the forward forms; do_ is dO.
 */
void oracle_prefill_backward(const double* q, const double* k, const double* v, const double* do_,
                             double* dq, double* dk, double* dv, long BH, long N, long d) {
    long bh;
#pragma omp parallel for schedule(dynamic)
    for (bh = 0; bh < BH; ++bh) {
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        const double* G = do_ + bh * N * d;
        double* DQ = dq + bh * N * d;
        double* DK = dk + bh * N * d;
        double* DV = dv + bh * N * d;
        memset(DQ, 0, (size_t)(N * d) * sizeof(double));
        memset(DK, 0, (size_t)(N * d) * sizeof(double));
        memset(DV, 0, (size_t)(N * d) * sizeof(double));
        for (long t = 0; t < N; ++t) {
            for (long s = 0; s <= t; s++) {
                double gv = 0.0, qk = 0.0;
                for (long c = 0; c < d; ++c) {
                    gv += G[t * d + c] * V[s * d + c];
                    qk += Q[t * d + c] * K[s * d + c];
                }
                for (long c = 0; c < d; ++c) {
                    DQ[t * d + c] += gv * K[s * d + c];
                    DK[s * d + c] += gv * Q[t * d + c];
                    DV[s * d + c] += qk * G[t * d + c];
                }
            }
        }
    }
}

/*
 * Block form with block size blk, in the order section 1 of the futurefh page
 * describes: for block i (rows [i*blk, min((i+1)*blk, N)) ),
 *     O_i = tril(Q_i K_i^T) V_i   (intra-block, left product)
 *         + Q_i S_{i-1}           (inter-block, right product)
 *     S_i = S_{i-1} + K_i^T V_i
 * with S_{-1} = 0.  The last block may be partial.  It exists to show that the
 * split is exact (it must agree with the two forms above).
 */
void oracle_prefill_blockwise(const double* q, const double* k, const double* v,
                              double* o, double* state_out, long BH, long N, long d,
                              long blk) {
    long bh;
#pragma omp parallel for schedule(dynamic)
    for (bh = 0; bh < BH; ++bh) {
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        double* O = o + bh * N * d;
        double* S = (double*)calloc((size_t)(d * d), sizeof(double));
        double* P = (double*)malloc((size_t)(blk * blk) * sizeof(double));
        for (long b0 = 0; b0 < N; b0 += blk) {
            long nb = (N - b0 < blk) ? (N - b0) : blk;
            /* P = tril(Q_i K_i^T), diagonal included */
            for (long r = 0; r < nb; ++r)
                for (long c = 0; c < nb; ++c) {
                    double acc = 0.0;
                    if (c <= r)
                        for (long x = 0; x < d; ++x) acc += Q[(b0 + r) * d + x] * K[(b0 + c) * d + x];
                    P[r * blk + c] = acc;
                }
            /* O_i = P V_i + Q_i S_{i-1} */
            for (long r = 0; r < nb; ++r)
                for (long j = 0; j < d; ++j) {
                    double intra = 0.0, inter = 0.0;
                    for (long c = 0; c < nb; ++c) intra += P[r * blk + c] * V[(b0 + c) * d + j];
                    for (long x = 0; x < d; ++x) inter += Q[(b0 + r) * d + x] * S[x * d + j];
                    O[(b0 + r) * d + j] = intra + inter;
                }
            /* S_i = S_{i-1} + K_i^T V_i */
            for (long x = 0; x < d; ++x)
                for (long j = 0; j < d; ++j) {
                    double acc = 0.0;
                    for (long c = 0; c < nb; ++c) acc += K[(b0 + c) * d + x] * V[(b0 + c) * d + j];
                    S[x * d + j] += acc;
                }
        }
        if (state_out) memcpy(state_out + bh * d * d, S, (size_t)(d * d) * sizeof(double));
        free(P);
        free(S);
    }
}

/*
 * One decode step (section 3 of the futurefh page runs decode separately from
 * prefill; the recurrence is the nabfollower page's fixed-size state):
 *     S <- S + k^T v ;  o = q S        (update first, then read)
 * q, k, v, o are [BH][d]; S is [BH][d][d] and is updated in place.
 */
void oracle_decode_step(const double* q, const double* k, const double* v,
                        double* S, double* o, long BH, long d) {
    long bh;
#pragma omp parallel for schedule(static)
    for (bh = 0; bh < BH; ++bh) {
        double* Sb = S + bh * d * d;
        const double* qb = q + bh * d;
        const double* kb = k + bh * d;
        const double* vb = v + bh * d;
        for (long i = 0; i < d; ++i)
            for (long j = 0; j < d; ++j) Sb[i * d + j] += kb[i] * vb[j];
        for (long j = 0; j < d; ++j) {
            double acc = 0.0;
            for (long i = 0; i < d; ++i) acc += qb[i] * Sb[i * d + j];
            o[bh * d + j] = acc;
        }
    }
}

/*
 * Packed variable-length prefill (data packing, section 4 of the futurefh
 * page): the recurrent form run separately on every sequence
 * [cu_seqlens[j], cu_seqlens[j+1]) of every head, the state starting at zero at
 * each sequence start.  q, k, v, o are [H][T][d]; state_out (may be NULL) is
 * [num_seqs][H][d][d].  An empty sequence leaves a zero state.
 * head_list (may be NULL = all heads) restricts the work to n_heads listed
 * heads; o and state_out are still indexed by the real head number.
 */
void oracle_prefill_varlen(const double* q, const double* k, const double* v,
                           const int* cu_seqlens, long num_seqs, long H, long T, long d,
                           double* o, double* state_out,
                           const int* head_list, long n_heads) {
    long nh = head_list ? n_heads : H;
    long item;
#pragma omp parallel for schedule(dynamic)
    for (item = 0; item < nh * num_seqs; ++item) {
        long h = head_list ? head_list[item / num_seqs] : item / num_seqs;
        long j = item % num_seqs;
        long t0 = cu_seqlens[j], t1 = cu_seqlens[j + 1];
        const double* Q = q + h * T * d;
        const double* K = k + h * T * d;
        const double* V = v + h * T * d;
        double* O = o + h * T * d;
        double* S = (double*)calloc((size_t)(d * d), sizeof(double));
        for (long t = t0; t < t1; ++t) {
            for (long i = 0; i < d; ++i)
                for (long c = 0; c < d; ++c) S[i * d + c] += K[t * d + i] * V[t * d + c];
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long i = 0; i < d; ++i) acc += Q[t * d + i] * S[i * d + c];
                O[t * d + c] = acc;
            }
        }
        if (state_out) memcpy(state_out + (j * H + h) * d * d, S, (size_t)(d * d) * sizeof(double));
        free(S);
    }
}

/*
 * Decode on an 8-bit state.  The yuliangy.com digest of the MiniMax-01 report
 * credits 8-bit quantisation with fitting more than a million tokens on one
 * eight-GPU machine; none of the pages gives a format.  The reading taken
 * here: row i of a head's state (key dimension i) is held as int8 codes c_ij
 * in [-127, 127] and one fp32 scale a_i, standing for S_ij = c_ij * a_i.
 *
 * Quantising one fp32 row x_0 .. x_{d-1}:
 *     m = max_j |x_j|
 *     if m < 2^-100:  a = 0 and every code is 0        (zero or negligible row)
 *     else:           a = m / 127,  c_j = nearest-even integer to x_j * (127 / m)
 * m / 127, 127 / m and x_j * (127 / m) are each one correctly rounded fp32
 * operation.  Codes are integer decisions, so they are taken in fp32 (the
 * precision the state is held in) and compared code for code with the kernel.
 */
static void quantize_row_q8(const float* x, signed char* c, float* a, long d) {
    float m = 0.0f;
    for (long j = 0; j < d; ++j) {
        const float ax = fabsf(x[j]);
        if (ax > m) m = ax;
    }
    if (m < 0x1p-100f) {
        *a = 0.0f;
        for (long j = 0; j < d; ++j) c[j] = 0;
        return;
    }
    const float inv = 127.0f / m;
    *a = m / 127.0f;
    for (long j = 0; j < d; ++j) {
        float r = rintf(x[j] * inv);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        c[j] = (signed char)r;
    }
}

/* rows x d fp32 states -> int8 codes [rows][d] and scales [rows]. */
void oracle_state_quantize_q8(const float* S, signed char* codes, float* scales, long rows, long d) {
    for (long r = 0; r < rows; ++r) quantize_row_q8(S + r * d, codes + r * d, scales + r, d);
}

/* codes [rows][d], scales [rows] -> S_ij = c_ij * a_i (one fp32 product). */
void oracle_state_dequantize_q8(const signed char* codes, const float* scales, float* S, long rows,
                                long d) {
    for (long r = 0; r < rows; ++r)
        for (long j = 0; j < d; ++j) S[r * d + j] = (float)codes[r * d + j] * scales[r];
}

/*
 * One decode step on the 8-bit state, update first and read second as in
 * oracle_decode_step:
 *     s_ij = fma(k_i, v_j, c_ij * a_i)    fp32: dequantise, then add k^T v
 *     o_j  = sum_i q_i s_ij              fp64 sum over the fp32 s
 *     codes, scales <- row-wise quantisation of s (above)
 * q, k, v are [BH][d] fp32 (bf16 inputs convert exactly); codes [BH][d][d]
 * and scales [BH][d] are updated in place; o is [BH][d].
 */
void oracle_decode_step_q8(const float* q, const float* k, const float* v, signed char* codes,
                           float* scales, double* o, long BH, long d) {
    long bh;
#pragma omp parallel for schedule(static)
    for (bh = 0; bh < BH; ++bh) {
        const float* qb = q + bh * d;
        const float* kb = k + bh * d;
        const float* vb = v + bh * d;
        signed char* cb = codes + bh * d * d;
        float* ab = scales + bh * d;
        float* s = (float*)malloc((size_t)(d * d) * sizeof(float));
        for (long i = 0; i < d; ++i)
            for (long j = 0; j < d; ++j) {
                const float deq = (float)cb[i * d + j] * ab[i];
                s[i * d + j] = fmaf(kb[i], vb[j], deq);
            }
        for (long j = 0; j < d; ++j) {
            double acc = 0.0;
            for (long i = 0; i < d; ++i) acc += (double)qb[i] * (double)s[i * d + j];
            o[bh * d + j] = acc;
        }
        for (long i = 0; i < d; ++i) quantize_row_q8(s + i * d, cb + i * d, ab + i, d);
        free(s);
    }
}
