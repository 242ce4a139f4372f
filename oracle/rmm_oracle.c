/*
 * rmm_oracle.c -- CPU oracle for Reduced Matrix Multiplication (RMM).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, the smoke check in __graft_entry__.py and the
 * CPU-baseline / reference legs of bench.py use it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Plain, single-threaded, obviously-correct C.  Floating-point arithmetic is
 * done in fp64 (inputs are bf16 bit patterns, widened exactly), except the
 * context-block score, which decides an integer set (see below).
 *
 * What it computes, and where it comes from:
 *
 *   Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
 *   LLM Inference (Lan, Li, Zhou), abstract: a training-free, input-adaptive
 *   method; each Transformer matrix product keeps the slices of its
 *   contraction dimension that the current input makes most significant, in
 *   a share set by one retention ratio r.
 *
 *   Input-adaptive matrix-product reduction for LLM inference (cf-1.com post):
 *     §2   the linear map Y = X @ W^T is replaced by Y ~= X @ W_sub^T over a
 *          subset of slices chosen from the current input; output shape is
 *          unchanged;
 *     §5.1 a cheap score computed from the current activations;
 *     §5.2 score -> top-k kept set;
 *     §5.3 gather activations and weights by the same kept set into compact
 *          operands and run a smaller dense product;
 *     §6.1 demo: top-k followed by a sort of the kept indices (stable order);
 *          keep ratio 1.0 reproduces the full product;
 *     §8   one common kept set for all tokens of a batch.
 *
 *   The score is fixed as s_h = max_t |X[t,h]| (exact, independent of the
 *   reduction order), the kept count as k = ceil(r*H) clamped to [1, H], and
 *   ties are broken toward the lower index, so the kept set is unique.
 *
 *   Attention: the same reduction applied to Q K^T along the head dimension
 *   (cf-1.com post §3.3: reduce inside a head, never drop whole heads), then
 *   an unreduced softmax(.) V.
 *
 *   Context-block attention (cf-1.com post §3.1): keys cut into blocks, a
 *   cheap per-block score, Q K^T on the kept blocks only.  Its kept-block
 *   decision is computed in single precision in a fixed order (stated at
 *   oracle_ctx_block_means); everything else stays fp64.
 *
 *   Decoder-layer glue: RMSNorm and SwiGLU as in Numerical Linear Algebra for
 *   Large Language Models (ai-feeds 2610.04631), Transformer component list.
 *
 * Error behaviour: every entry point returns 0 on success, a negative value
 * on an invalid argument, and ORACLE_ERR_NONFINITE if an input holds a NaN or
 * an infinity (the method is only defined on finite inputs).
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_NONFINITE (-2)
#define ORACLE_ERR_NOMEM (-3)

/* ---- bf16 helpers -------------------------------------------------------- */

int oracle_ctx_select(const float* scores, long nblk, long kc, int32_t* blocks);

static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int bf16_is_finite(uint16_t b) { return (b & 0x7F80u) != 0x7F80u; }

static int all_finite(const uint16_t* p, long n) {
    for (long i = 0; i < n; ++i)
        if (!bf16_is_finite(p[i])) return 0;
    return 1;
}

/* |x| of a finite bf16 value, as an integer that orders like |x|:
 * clearing the sign bit leaves exponent:mantissa, which is monotone in the
 * magnitude for finite values, and maps -0 and +0 to the same key 0. */
static uint16_t bf16_magnitude_key(uint16_t b) { return (uint16_t)(b & 0x7FFFu); }

/* ---- k = ceil(r*H) ------------------------------------------------------- */

/* Number of kept contraction slices for retention ratio r (abstract: one
 * retention-ratio knob).  r must lie in (0, 1]; the result is ceil(r*H)
 * evaluated in double and clamped to [1, H].  Returns -1 for a bad r or H. */
int oracle_k_for(long H, double r) {
    if (!(H >= 1) || !(r > 0.0) || !(r <= 1.0)) return -1;
    double kk = ceil(r * (double)H);
    long k = (long)kk;
    if (k < 1) k = 1;
    if (k > H) k = H;
    return (int)k;
}

/* ---- §5.1 score ---------------------------------------------------------- */

/* s[h] = max over t of |X[t,h]|, returned as the magnitude key (sign bit
 * cleared).  X is [T, H] row-major bf16.  With T == 0 every score is 0. */
int oracle_score(const uint16_t* X, long T, long H, uint16_t* s) {
    if (H < 1 || T < 0 || !s || (T > 0 && !X)) return ORACLE_ERR_ARG;
    if (!all_finite(X, T * H)) return ORACLE_ERR_NONFINITE;
    for (long h = 0; h < H; ++h) s[h] = 0;
    for (long t = 0; t < T; ++t)
        for (long h = 0; h < H; ++h) {
            uint16_t m = bf16_magnitude_key(X[t * H + h]);
            if (m > s[h]) s[h] = m;
        }
    return 0;
}

/* ---- §5.2 select --------------------------------------------------------- */

typedef struct {
    uint16_t score;
    int32_t index;
} keyed;

/* Total order of the kept-set rule: larger score first; for equal scores the
 * lower index first. */
static int better_first(const void* a, const void* b) {
    const keyed* x = (const keyed*)a;
    const keyed* y = (const keyed*)b;
    if (x->score != y->score) return (x->score > y->score) ? -1 : 1;
    return (x->index < y->index) ? -1 : (x->index > y->index) ? 1 : 0;
}

static int ascending_int(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x < y) ? -1 : (x > y) ? 1 : 0;
}

/* Top-k of s under (score desc, index asc), emitted in ascending index order
 * (the demo's sort after top-k keeps the kept slices in their original
 * order).  idx receives k entries. */
int oracle_select(const uint16_t* s, long H, long k, int32_t* idx) {
    if (!s || !idx || H < 1 || k < 1 || k > H) return ORACLE_ERR_ARG;
    keyed* all = (keyed*)malloc(sizeof(keyed) * (size_t)H);
    if (!all) return ORACLE_ERR_NOMEM;
    for (long h = 0; h < H; ++h) {
        all[h].score = s[h];
        all[h].index = (int32_t)h;
    }
    qsort(all, (size_t)H, sizeof(keyed), better_first);
    for (long j = 0; j < k; ++j) idx[j] = all[j].index;
    free(all);
    qsort(idx, (size_t)k, sizeof(int32_t), ascending_int);
    return 0;
}

/* ---- §5.3 gather + smaller dense product ---------------------------------- */

/* Y[r, c] = sum over j < k of X[t_r, idx[j]] * W[n_c, idx[j]], in fp64,
 * summed over ascending j.  X is [T, H], W is [N, H] (the layer's weight as
 * stored by the model: one row per output feature).  rows selects which
 * token rows t_r to compute (NULL: all T rows, in order) and cols which
 * output features n_c (NULL: all N, in order); Y is [nrows, ncols].
 * idx may hold any list of distinct in-range indices (used by the tests to
 * form complementary sets). */
int oracle_reduced_product(const uint16_t* X, const uint16_t* W, long T, long H, long N,
                           const int32_t* idx, long k, const int64_t* rows, long nrows,
                           const int64_t* cols, long ncols, double* Y) {
    if (!X || !W || !idx || !Y || T < 1 || H < 1 || N < 1 || k < 1 || k > H) return ORACLE_ERR_ARG;
    if (!rows) nrows = T;
    if (!cols) ncols = N;
    if (nrows < 0 || ncols < 0) return ORACLE_ERR_ARG;
    for (long j = 0; j < k; ++j)
        if (idx[j] < 0 || idx[j] >= H) return ORACLE_ERR_ARG;
    for (long r = 0; r < nrows; ++r)
        if (rows && (rows[r] < 0 || rows[r] >= T)) return ORACLE_ERR_ARG;
    for (long c = 0; c < ncols; ++c)
        if (cols && (cols[c] < 0 || cols[c] >= N)) return ORACLE_ERR_ARG;
    if (!all_finite(X, T * H) || !all_finite(W, N * H)) return ORACLE_ERR_NONFINITE;

    /* One output row per iteration; with the OpenMP build (the parallel CPU
     * baseline) rows are spread over the host's threads, each row still
     * computed by one thread in the order below, so the results are the
     * same bits as the single-threaded build's. */
    int nomem = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : nomem)
    for (long r = 0; r < nrows; ++r) {
        double* xk = (double*)malloc(sizeof(double) * (size_t)k);
        double* wk = (double*)malloc(sizeof(double) * (size_t)k);
        if (!xk || !wk) {
            nomem = 1;
        } else {
            long t = rows ? (long)rows[r] : r;
            /* gather the kept slices of this activation row */
            for (long j = 0; j < k; ++j) xk[j] = bf16_to_double(X[t * H + idx[j]]);
            for (long c = 0; c < ncols; ++c) {
                long n = cols ? (long)cols[c] : c;
                /* gather the same kept slices of the weight row, then the smaller dot product */
                for (long j = 0; j < k; ++j) wk[j] = bf16_to_double(W[n * H + idx[j]]);
                double acc = 0.0;
                for (long j = 0; j < k; ++j) acc += xk[j] * wk[j];
                Y[r * ncols + c] = acc;
            }
        }
        free(xk);
        free(wk);
    }
    return nomem ? ORACLE_ERR_NOMEM : 0;
}

/* Threads the product loop may use: 1 in the plain build. */
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- block-granular kept sets (§5.2, §6.1 demo) ------------------------ */

/* The kept set chosen per block of `block` consecutive contraction slices
 * (the demo keeps 64-wide blocks of the down projection's input, scored from
 * the current activation, top-k of the block scores, sorted).  Block j covers
 * slices [j*block, (j+1)*block); its score is the largest of its slices'
 * scores s (max keeps the score exact and independent of any summation
 * order, as the per-slice score is).  The kb best blocks under (score desc,
 * block index asc) are written to blocks in ascending order.  H must be a
 * multiple of block. */
int oracle_block_select(const uint16_t* s, long H, long block, long kb, int32_t* blocks) {
    if (!s || !blocks || block < 1 || H < block || H % block != 0) return ORACLE_ERR_ARG;
    long nb = H / block;
    if (kb < 1 || kb > nb) return ORACLE_ERR_ARG;
    uint16_t* bs = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)nb);
    if (!bs) return ORACLE_ERR_NOMEM;
    for (long j = 0; j < nb; ++j) {
        uint16_t m = 0;
        for (long i = 0; i < block; ++i)
            if (s[j * block + i] > m) m = s[j * block + i];
        bs[j] = m;
    }
    int rc = oracle_select(bs, nb, kb, blocks);
    free(bs);
    return rc;
}

/* Block-granular kept set scored by the mean magnitude of the block, the
 * score of the FFN demo in the cf-1.com post (§5.1: a block's importance is
 * its mean absolute activation; §6.1: blocks of 64 of the FFN intermediate
 * dimension, top blocks by that mean, sorted).  The score decides an integer
 * set, so it is computed in single precision in one stated order: the sum
 * runs over the tokens t ascending and, within a token, over the block's
 * slices ascending (float additions from 0), then one correctly rounded
 * division by T*block.  The kb best blocks under (score desc, block index
 * asc) are written to blocks in ascending order. */
int oracle_block_select_mean(const uint16_t* X, long T, long H, long block, long kb, int32_t* blocks) {
    if (!X || !blocks || T < 1 || block < 1 || H < block || H % block != 0) return ORACLE_ERR_ARG;
    long nb = H / block;
    if (kb < 1 || kb > nb) return ORACLE_ERR_ARG;
    if (!all_finite(X, T * H)) return ORACLE_ERR_NONFINITE;
    float* bs = (float*)malloc(sizeof(float) * (size_t)nb);
    if (!bs) return ORACLE_ERR_NOMEM;
    for (long j = 0; j < nb; ++j) {
        float sum = 0.0f;
        for (long t = 0; t < T; ++t)
            for (long i = 0; i < block; ++i) sum += fabsf((float)bf16_to_double(X[t * H + j * block + i]));
        bs[j] = sum / (float)(T * block);
    }
    int rc = oracle_ctx_select(bs, nb, kb, blocks);
    free(bs);
    return rc;
}

/* The whole reduced linear map: k = ceil(r*H); score; select; gather and
 * product.  idx_out (k entries, may be NULL) receives the kept set. */
int oracle_linear(const uint16_t* X, const uint16_t* W, long T, long H, long N, double r,
                  const int64_t* rows, long nrows, const int64_t* cols, long ncols, double* Y,
                  int32_t* idx_out) {
    int k = oracle_k_for(H, r);
    if (k < 1) return ORACLE_ERR_ARG;
    if (!X || !W || !Y || T < 1 || N < 1) return ORACLE_ERR_ARG;
    uint16_t* s = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)H);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    if (!s || !idx) {
        free(s);
        free(idx);
        return ORACLE_ERR_NOMEM;
    }
    int rc = oracle_score(X, T, H, s);
    if (rc == 0) rc = oracle_select(s, H, k, idx);
    if (rc == 0) rc = oracle_reduced_product(X, W, T, H, N, idx, k, rows, nrows, cols, ncols, Y);
    if (rc == 0 && idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)k);
    free(s);
    free(idx);
    return rc;
}

/* ---- attention: Q K^T reduced along the head dimension, then softmax . V -- */

/* Q [B, Hq, T, d], K [B, Hkv, L, d], V [B, Hkv, L, d] (bf16, keys stored one
 * row per position), O [B, Hq, nrows, d] (fp64).
 *
 * Kept set: per (b, KV head g) over the stacked queries of g's group
 * (per_query_head == 0), or per (b, query head) (per_query_head == 1):
 *   s_j = max over the group's heads q and all t < T of |Q[b,q,t,j]|, j < d;
 *   S   = top-k of s under (score desc, index asc), ascending.
 * Logits: logit[l] = scale * sum over j in S of Q[b,q,t,j] * K[b,g,l,j].
 * Query t sits at position L - T + t; with causal != 0 keys l > L - T + t are
 * masked out.  Softmax in fp64 (max-subtracted), O = sum_l p_l V[b,g,l,:].
 * idx_out: [B, Hkv, k] (or [B, Hq, k] per query head), may be NULL.
 * t_rows (NULL: all T) lists the query rows to compute; the kept set always
 * uses all T rows.  idx_in (NULL: select as above) supplies the kept sets
 * instead, laid out like idx_out -- for a layer oracle that follows the index
 * sets another implementation chose, so that a near-tie in an upstream input
 * cannot make the two compute different products. */
/* The attention of one call.  key_keep (NULL: every key) is a 0/1 mask
 * [B][nsets][L]: the keys a set's query rows may attend to (the context-block
 * reduction below); a row that may attend to no key gets a zero output. */
static int attention_core(const uint16_t* Q, const uint16_t* K, const uint16_t* V, long B, long Hq,
                          long Hkv, long T, long L, long d, long k, int causal, double scale,
                          int per_query_head, const int64_t* t_rows, long nrows, double* O,
                          int32_t* idx_out, const int32_t* idx_in, const uint8_t* key_keep) {
    if (!Q || !K || !V || !O || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < T || d < 1 || k < 1 ||
        k > d || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    if (!t_rows) nrows = T;
    if (!all_finite(Q, B * Hq * T * d) || !all_finite(K, B * Hkv * L * d) ||
        !all_finite(V, B * Hkv * L * d))
        return ORACLE_ERR_NONFINITE;
    long G = Hq / Hkv;
    long nsets = per_query_head ? Hq : Hkv;
    uint16_t* s = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)d);
    int32_t* S = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* logit = (double*)malloc(sizeof(double) * (size_t)L);
    if (!s || !S || !logit) {
        free(s);
        free(S);
        free(logit);
        return ORACLE_ERR_NOMEM;
    }
    int rc = 0;
    for (long b = 0; b < B && rc == 0; ++b) {
        for (long set = 0; set < nsets && rc == 0; ++set) {
            long q_lo = per_query_head ? set : set * G;
            long q_hi = per_query_head ? set + 1 : (set + 1) * G;
            long g = per_query_head ? set / G : set;
            if (idx_in) {
                /* the given kept set */
                memcpy(S, idx_in + (b * nsets + set) * k, sizeof(int32_t) * (size_t)k);
                for (long j = 0; j < k; ++j)
                    if (S[j] < 0 || S[j] >= d) rc = ORACLE_ERR_ARG;
                if (rc) break;
            } else {
                /* score over the set's stacked query rows */
                for (long j = 0; j < d; ++j) s[j] = 0;
                for (long q = q_lo; q < q_hi; ++q)
                    for (long t = 0; t < T; ++t)
                        for (long j = 0; j < d; ++j) {
                            uint16_t m = bf16_magnitude_key(Q[((b * Hq + q) * T + t) * d + j]);
                            if (m > s[j]) s[j] = m;
                        }
                rc = oracle_select(s, d, k, S);
                if (rc) break;
            }
            if (idx_out) memcpy(idx_out + (b * nsets + set) * k, S, sizeof(int32_t) * (size_t)k);
            const uint16_t* Kg = K + (b * Hkv + g) * L * d;
            const uint16_t* Vg = V + (b * Hkv + g) * L * d;
            for (long q = q_lo; q < q_hi; ++q) {
                for (long r = 0; r < nrows; ++r) {
                    long t = t_rows ? (long)t_rows[r] : r;
                    if (t < 0 || t >= T) {
                        rc = ORACLE_ERR_ARG;
                        break;
                    }
                    const uint16_t* qv = Q + ((b * Hq + q) * T + t) * d;
                    const uint8_t* kk = key_keep ? key_keep + (b * nsets + set) * L : NULL;
                    long last = causal ? (L - T + t) : (L - 1);
                    double mx = -INFINITY;
                    for (long l = 0; l <= last; ++l) {
                        if (kk && !kk[l]) continue;
                        double acc = 0.0;
                        for (long j = 0; j < k; ++j)
                            acc += bf16_to_double(qv[S[j]]) * bf16_to_double(Kg[l * d + S[j]]);
                        logit[l] = scale * acc;
                        if (logit[l] > mx) mx = logit[l];
                    }
                    double den = 0.0;
                    for (long l = 0; l <= last; ++l) {
                        if (kk && !kk[l]) continue;
                        logit[l] = exp(logit[l] - mx);
                        den += logit[l];
                    }
                    double* o = O + ((b * Hq + q) * nrows + r) * d;
                    for (long c = 0; c < d; ++c) {
                        double acc = 0.0;
                        for (long l = 0; l <= last; ++l)
                            if (!kk || kk[l]) acc += logit[l] * bf16_to_double(Vg[l * d + c]);
                        o[c] = den > 0.0 ? acc / den : 0.0;
                    }
                }
            }
        }
    }
    free(s);
    free(S);
    free(logit);
    return rc;
}

int oracle_attention(const uint16_t* Q, const uint16_t* K, const uint16_t* V, long B, long Hq,
                     long Hkv, long T, long L, long d, long k, int causal, double scale,
                     int per_query_head, const int64_t* t_rows, long nrows, double* O,
                     int32_t* idx_out, const int32_t* idx_in) {
    return attention_core(Q, K, V, B, Hq, Hkv, T, L, d, k, causal, scale, per_query_head, t_rows, nrows, O,
                          idx_out, idx_in, NULL);
}

/* ---- context-block reduction of Q K^T (sequence direction) ----------------
 *
 * Input-adaptive matrix-product reduction for LLM inference (cf-1.com post),
 * §3.1: during generation the keys are cut into blocks of consecutive
 * positions, a cheap score tells which blocks may draw real attention, and
 * the full Q K^T runs on the kept blocks only; §7: the gain grows with the
 * context.  The pages fix neither the cheap score nor the kept count; the
 * readings taken here:
 *   - block j holds the positions [j*bc, min(L, (j+1)*bc));
 *   - its summary is its mean key  mean_j[c] = (sum over its l of K[l,c]) / n_j;
 *   - its score for a kept set (a KV head's stacked query rows, or one query
 *     head's rows) is the largest dot product of one of the set's query rows
 *     with mean_j;
 *   - kc = ceil(r_ctx * nblk) blocks are kept under (score desc, index asc),
 *     listed in ascending order;
 *   - keys of dropped blocks take no part in the softmax.
 * Summary and score decide which blocks are kept, so they are computed in
 * single precision in one fixed order, the precision and order in which the
 * GPU path takes the same decision:
 *   sum  : float additions over l ascending, starting from 0;
 *   mean : sum / (float)n_j (correctly rounded division);
 *   dot  : fmaf chain over c ascending, starting from 0. */

static float bf16_to_float(uint16_t b) { return (float)bf16_to_double(b); }

/* means [B][Hkv][nblk][d], nblk = ceil(L / bc); K [B][Hkv][L][d]. */
int oracle_ctx_block_means(const uint16_t* K, long B, long Hkv, long L, long d, long bc, float* means) {
    if (!K || !means || B < 1 || Hkv < 1 || L < 1 || d < 1 || bc < 1) return ORACLE_ERR_ARG;
    if (!all_finite(K, B * Hkv * L * d)) return ORACLE_ERR_NONFINITE;
    long nblk = (L + bc - 1) / bc;
    for (long b = 0; b < B; ++b)
        for (long g = 0; g < Hkv; ++g) {
            const uint16_t* Kg = K + (b * Hkv + g) * L * d;
            for (long j = 0; j < nblk; ++j) {
                long l0 = j * bc, l1 = l0 + bc < L ? l0 + bc : L;
                for (long c = 0; c < d; ++c) {
                    float sum = 0.0f;
                    for (long l = l0; l < l1; ++l) sum += bf16_to_float(Kg[l * d + c]);
                    means[((b * Hkv + g) * nblk + j) * d + c] = sum / (float)(l1 - l0);
                }
            }
        }
    return 0;
}

/* scores [B][nsets][nblk] from Q [B][Hq][T][d] and the block means. */
int oracle_ctx_block_scores(const uint16_t* Q, const float* means, long B, long Hq, long Hkv, long T,
                            long nblk, long d, int per_query_head, float* scores) {
    if (!Q || !means || !scores || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || nblk < 1 || d < 1 ||
        Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    if (!all_finite(Q, B * Hq * T * d)) return ORACLE_ERR_NONFINITE;
    long G = Hq / Hkv;
    long nsets = per_query_head ? Hq : Hkv;
    for (long b = 0; b < B; ++b)
        for (long set = 0; set < nsets; ++set) {
            long q_lo = per_query_head ? set : set * G;
            long q_hi = per_query_head ? set + 1 : (set + 1) * G;
            long g = per_query_head ? set / G : set;
            for (long j = 0; j < nblk; ++j) {
                const float* m = means + ((b * Hkv + g) * nblk + j) * d;
                float best = -INFINITY;
                for (long q = q_lo; q < q_hi; ++q)
                    for (long t = 0; t < T; ++t) {
                        const uint16_t* qv = Q + ((b * Hq + q) * T + t) * d;
                        float acc = 0.0f;
                        for (long c = 0; c < d; ++c) acc = fmaf(bf16_to_float(qv[c]), m[c], acc);
                        if (acc > best) best = acc;
                    }
                scores[(b * nsets + set) * nblk + j] = best;
            }
        }
    return 0;
}

typedef struct {
    float score;
    int32_t index;
} fkeyed;

static int fbetter_first(const void* a, const void* b) {
    const fkeyed* x = (const fkeyed*)a;
    const fkeyed* y = (const fkeyed*)b;
    if (x->score != y->score) return x->score > y->score ? -1 : 1;
    return x->index < y->index ? -1 : (x->index > y->index ? 1 : 0);
}

/* The kc best of nblk block scores under (score desc, index asc), ascending. */
int oracle_ctx_select(const float* scores, long nblk, long kc, int32_t* blocks) {
    if (!scores || !blocks || nblk < 1 || kc < 1 || kc > nblk) return ORACLE_ERR_ARG;
    fkeyed* all = (fkeyed*)malloc(sizeof(fkeyed) * (size_t)nblk);
    if (!all) return ORACLE_ERR_NOMEM;
    for (long j = 0; j < nblk; ++j) {
        if (isnan(scores[j])) {
            free(all);
            return ORACLE_ERR_NONFINITE;
        }
        all[j].score = scores[j];
        all[j].index = (int32_t)j;
    }
    qsort(all, (size_t)nblk, sizeof(fkeyed), fbetter_first);
    for (long j = 0; j < kc; ++j) blocks[j] = all[j].index;
    free(all);
    qsort(blocks, (size_t)kc, sizeof(int32_t), ascending_int);
    return 0;
}

/* Attention with both reductions: the kept head dimensions (k of d, as in
 * oracle_attention) and the kept context blocks (kc of ceil(L/bc) blocks of
 * bc keys).  blocks_in ([B][nsets][kc], NULL: select them as above) and
 * idx_in ([B][nsets][k], NULL: select from Q) supply given sets; blocks_out
 * and idx_out (may be NULL) receive the sets used. */
int oracle_attention_ctx(const uint16_t* Q, const uint16_t* K, const uint16_t* V, long B, long Hq,
                         long Hkv, long T, long L, long d, long k, int causal, double scale,
                         int per_query_head, long bc, long kc, const int64_t* t_rows, long nrows,
                         double* O, int32_t* idx_out, int32_t* blocks_out, const int32_t* idx_in,
                         const int32_t* blocks_in) {
    if (!Q || !K || !V || !O || B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < T || d < 1 || bc < 1 ||
        Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    long nblk = (L + bc - 1) / bc;
    if (kc < 1 || kc > nblk) return ORACLE_ERR_ARG;
    long nsets = per_query_head ? Hq : Hkv;
    int32_t* blocks = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B * nsets * kc));
    uint8_t* keep = (uint8_t*)calloc((size_t)(B * nsets * L), 1);
    float* means = NULL;
    float* scores = NULL;
    int rc = (blocks && keep) ? 0 : ORACLE_ERR_NOMEM;
    if (rc == 0 && blocks_in) {
        memcpy(blocks, blocks_in, sizeof(int32_t) * (size_t)(B * nsets * kc));
        for (long i = 0; i < B * nsets * kc; ++i)
            if (blocks[i] < 0 || blocks[i] >= nblk) rc = ORACLE_ERR_ARG;
    } else if (rc == 0) {
        means = (float*)malloc(sizeof(float) * (size_t)(B * Hkv * nblk * d));
        scores = (float*)malloc(sizeof(float) * (size_t)(B * nsets * nblk));
        if (!means || !scores) rc = ORACLE_ERR_NOMEM;
        if (rc == 0) rc = oracle_ctx_block_means(K, B, Hkv, L, d, bc, means);
        if (rc == 0) rc = oracle_ctx_block_scores(Q, means, B, Hq, Hkv, T, nblk, d, per_query_head, scores);
        for (long i = 0; rc == 0 && i < B * nsets; ++i)
            rc = oracle_ctx_select(scores + i * nblk, nblk, kc, blocks + i * kc);
    }
    for (long i = 0; rc == 0 && i < B * nsets; ++i)
        for (long j = 0; j < kc; ++j) {
            long l0 = (long)blocks[i * kc + j] * bc, l1 = l0 + bc < L ? l0 + bc : L;
            for (long l = l0; l < l1; ++l) keep[i * L + l] = 1;
        }
    if (rc == 0 && blocks_out) memcpy(blocks_out, blocks, sizeof(int32_t) * (size_t)(B * nsets * kc));
    if (rc == 0)
        rc = attention_core(Q, K, V, B, Hq, Hkv, T, L, d, k, causal, scale, per_query_head, t_rows, nrows, O,
                            idx_out, idx_in, keep);
    free(blocks);
    free(keep);
    free(means);
    free(scores);
    return rc;
}


/* y[t,:] = x[t,:] / sqrt(mean_h x[t,h]^2 + eps)  (norm weight 1). */
int oracle_rmsnorm(const uint16_t* x, long T, long H, double eps, double* y) {
    if (!x || !y || T < 1 || H < 1) return ORACLE_ERR_ARG;
    if (!all_finite(x, T * H)) return ORACLE_ERR_NONFINITE;
    for (long t = 0; t < T; ++t) {
        double ss = 0.0;
        for (long h = 0; h < H; ++h) {
            double v = bf16_to_double(x[t * H + h]);
            ss += v * v;
        }
        double inv = 1.0 / sqrt(ss / (double)H + eps);
        for (long h = 0; h < H; ++h) y[t * H + h] = bf16_to_double(x[t * H + h]) * inv;
    }
    return 0;
}

/* out = silu(g) * u elementwise, silu(z) = z / (1 + exp(-z)). */
int oracle_swiglu(const uint16_t* g, const uint16_t* u, long n, double* out) {
    if (!g || !u || !out || n < 1) return ORACLE_ERR_ARG;
    if (!all_finite(g, n) || !all_finite(u, n)) return ORACLE_ERR_NONFINITE;
    for (long i = 0; i < n; ++i) {
        double z = bf16_to_double(g[i]);
        out[i] = z / (1.0 + exp(-z)) * bf16_to_double(u[i]);
    }
    return 0;
}
