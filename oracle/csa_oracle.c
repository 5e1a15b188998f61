/*
 * csa_oracle.c -- CPU oracle for the CSA lightning-indexer top-k step.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * definition that the CUDA path is checked against.  Only the tests, the
 * package's smoke check and the bench's CPU-baseline leg may load it; the
 * product path never does.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What it computes (written out from the definition, fp64 accumulation):
 *
 *   For every batch b and query row i (absolute position t = i + q_offset):
 *     visible set  V = { s in [0,T) : !causal  or  (s+1)*m - 1 <= t }
 *       -- compressed key s summarises tokens [s*m, (s+1)*m); it is usable
 *          once its last token is at or before t.  ("StreamIndex:
 *          Memory-Bounded Compressed Sparse Attention via Streaming Top-k",
 *          abstract: keys are compressed at ratio m=4 and scored per query.)
 *     score        I[t,s] = sum_h w[t,h] * ReLU( sum_j q[t,h,j] * k[s,j] )
 *       -- the lightning indexer: a dot product of each indexer head's query
 *          with the compressed key, ReLU, then a head-weighted sum
 *          ("StreamIndex ...", abstract: "a learned scoring projection over
 *          compressed keys"; "FlashMemory-DeepSeek-V4: Lightning Index
 *          Ultra-Long Context via Lookahead Sparse Attention", axioms:
 *          a dot product with compressed chunk summaries fused across heads
 *          with ReLU).  No further scale: any scale lives in w.
 *     FP8 keys     k[s,j] = k_scale[s] * E4M3(k8[s,j])   (exact in fp64)
 *     selection
 *       mode 0 (ReLU top-k): order V by (I descending, s ascending) and keep
 *         the first min(topk, |V|) -- "StreamIndex ...", abstract: the top-k
 *         are selected per query; ties go to the lower index.
 *       mode 1 (sigmoid gate): keep s in V with sigmoid(I) > 0.5, which holds
 *         exactly when I > 0, then keep at most topk of them by the same
 *         order -- "FlashMemory-DeepSeek-V4 ...", "What carries the
 *         argument": a sigmoid replaces the ReLU's role in selection and a
 *         fixed 0.5 threshold replaces the fixed top-k.
 *     output       slots [0, n) hold (s, (float)I) in that order; slots
 *                  [n, topk) hold (-1, -inf).  A zero score is written as
 *                  +0.0.
 *
 * Input formats are decoded from their definitions: bfloat16 is the upper 16
 * bits of an IEEE-754 binary32; E4M3 ("fn" variant of the OCP 8-bit floating
 * point format) has 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits, subnormals at exponent 0, no infinities, and NaN only at S.1111.111.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* bfloat16 bits -> value: the bits are the high half of a binary32. */
double csa_oracle_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E4M3 ("fn") byte -> value, from the format definition. */
double csa_oracle_e4m3_value(uint8_t byte)
{
    int sign = (byte >> 7) & 1;
    int expo = (byte >> 3) & 0xF;
    int mant = byte & 0x7;
    double v;
    if (expo == 0xF && mant == 0x7)
        return NAN;
    if (expo == 0)
        v = ldexp((double)mant / 8.0, 1 - 7);          /* subnormal */
    else
        v = ldexp(1.0 + (double)mant / 8.0, expo - 7); /* normal */
    return sign ? -v : v;
}

/* The absolute position of query row i: rows are aligned so that the last
 * query sits at the end of the keys' token span unless told otherwise. */
static long long query_position(long long i, long long q_offset)
{
    return i + q_offset;
}

static int key_visible(long long s, long long t, int m, int causal)
{
    if (!causal)
        return 1;
    return (s + 1) * (long long)m - 1 <= t;
}

typedef struct {
    double score;
    int32_t index;
} cand_t;

/* Order: higher score first; equal scores -> lower index first. */
static int cand_order(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa;
    const cand_t *b = (const cand_t *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    if (a->index < b->index) return -1;
    if (a->index > b->index) return 1;
    return 0;
}

/* Decode the keys of batch b into fp64 (the effective key values). */
static void decode_keys(const void *k, const float *k_scale, int key_fmt,
                        int b, int T, int d, double *keff)
{
    long long base = (long long)b * T * d;
    for (long long s = 0; s < T; ++s) {
        for (int j = 0; j < d; ++j) {
            long long e = base + s * d + j;
            double v;
            if (key_fmt == 0)
                v = csa_oracle_bf16_value(((const uint16_t *)k)[e]);
            else
                v = (double)k_scale[(long long)b * T + s] *
                    csa_oracle_e4m3_value(((const uint8_t *)k)[e]);
            keff[s * d + j] = v;
        }
    }
}

/* I[t,s] for one query row against one (decoded) key, straight from the
 * definition. */
static double indexer_score(const double *qrow /* [H,d] */, const float *wrow /* [H] */,
                            const double *key /* [d] */, int H, int d)
{
    double total = 0.0;
    for (int h = 0; h < H; ++h) {
        double logit = 0.0;
        for (int j = 0; j < d; ++j)
            logit += qrow[(long long)h * d + j] * key[j];
        double relu = logit > 0.0 ? logit : 0.0;
        total += (double)wrow[h] * relu;
    }
    return total + 0.0; /* -0.0 -> +0.0 */
}

static int check_args(int key_fmt, const float *k_scale, int B, int S, int T, int H,
                      int d, int m, int topk, int mode)
{
    if (B < 0 || S < 0 || T < 0 || H <= 0 || d <= 0 || m <= 0 || topk <= 0)
        return ORACLE_ERR_ARG;
    if (key_fmt != 0 && key_fmt != 1)
        return ORACLE_ERR_ARG;
    if (key_fmt == 1 && k_scale == NULL)
        return ORACLE_ERR_ARG;
    if (mode != 0 && mode != 1)
        return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

/*
 * All indexer scores of one query row (b, i): out[s] = I[t,s] for every key
 * s < T (visible or not), and vis[s] = 1 iff s is causally visible.
 */
int csa_oracle_score_row(const uint16_t *q, const float *w, const void *k,
                         const float *k_scale, int key_fmt, int B, int S, int T,
                         int H, int d, int m, int causal, long long q_offset,
                         int b, long long i, double *out, int32_t *vis)
{
    if (check_args(key_fmt, k_scale, B, S, T, H, d, m, 1, 0) != ORACLE_OK)
        return ORACLE_ERR_ARG;
    if (b < 0 || b >= B || i < 0 || i >= S)
        return ORACLE_ERR_ARG;
    double *keff = (double *)malloc(sizeof(double) * (size_t)T * (size_t)d + 8);
    double *qrow = (double *)malloc(sizeof(double) * (size_t)H * (size_t)d);
    if (!keff || !qrow) {
        free(keff);
        free(qrow);
        return ORACLE_ERR_NOMEM;
    }
    decode_keys(k, k_scale, key_fmt, b, T, d, keff);
    long long row = (long long)b * S + i;
    for (long long e = 0; e < (long long)H * d; ++e)
        qrow[e] = csa_oracle_bf16_value(q[row * H * d + e]);
    long long t = query_position(i, q_offset);
    for (long long s = 0; s < T; ++s) {
        out[s] = indexer_score(qrow, w + row * H, keff + s * d, H, d);
        vis[s] = key_visible(s, t, m, causal);
    }
    free(keff);
    free(qrow);
    return ORACLE_OK;
}

/*
 * Top-k (mode 0) or gated (mode 1) selection for a list of query rows.
 *
 *   rows:      n_rows flat row ids r = b*S + i, or NULL for all B*S rows in order
 *   out_idx:   [n_rows, topk] int32
 *   out_score: [n_rows, topk] float  (the fp64 score rounded once)
 *   out_score64: optional [n_rows, topk] double (the fp64 score; NaN on padding)
 *   out_count: optional [n_rows] int32, the number of filled slots
 *
 * OpenMP parallelises over query rows; each row is computed exactly as the
 * header describes.  Keys are decoded once per batch.
 */
int csa_oracle_topk(const uint16_t *q, const float *w, const void *k,
                    const float *k_scale, int key_fmt, int B, int S, int T, int H,
                    int d, int m, int topk, int causal, int mode, long long q_offset,
                    const int64_t *rows, long long n_rows, int32_t *out_idx,
                    float *out_score, double *out_score64, int32_t *out_count)
{
    int rc = check_args(key_fmt, k_scale, B, S, T, H, d, m, topk, mode);
    if (rc != ORACLE_OK)
        return rc;
    if (rows == NULL)
        n_rows = (long long)B * S;
    for (long long r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (long long)B * S)
            return ORACLE_ERR_ARG;

    double *keff = (double *)malloc(sizeof(double) * (size_t)T * (size_t)d + 8);
    if (!keff)
        return ORACLE_ERR_NOMEM;
    int status = ORACLE_OK;

    for (int b = 0; b < B && status == ORACLE_OK; ++b) {
        /* Skip batches none of the requested rows belong to. */
        int needed = rows == NULL;
        for (long long r = 0; !needed && r < n_rows; ++r)
            needed = rows[r] / S == b;
        if (!needed)
            continue;
        decode_keys(k, k_scale, key_fmt, b, T, d, keff);

#pragma omp parallel
        {
            double *qrow = (double *)malloc(sizeof(double) * (size_t)H * (size_t)d);
            cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)T + sizeof(cand_t));
            if (!qrow || !cand) {
#pragma omp critical
                status = ORACLE_ERR_NOMEM;
            } else {
#pragma omp for schedule(dynamic, 1)
                for (long long r = 0; r < n_rows; ++r) {
                    long long row = rows ? rows[r] : r;
                    if (row / S != b)
                        continue;
                    long long i = row % S;
                    long long t = query_position(i, q_offset);
                    for (long long e = 0; e < (long long)H * d; ++e)
                        qrow[e] = csa_oracle_bf16_value(q[row * H * d + e]);
                    const float *wrow = w + row * H;

                    long long n = 0;
                    for (long long s = 0; s < T; ++s) {
                        if (!key_visible(s, t, m, causal))
                            continue;
                        double I = indexer_score(qrow, wrow, keff + s * d, H, d);
                        if (mode == 1 && !(I > 0.0)) /* sigmoid(I) > 0.5 <=> I > 0 */
                            continue;
                        cand[n].score = I;
                        cand[n].index = (int32_t)s;
                        ++n;
                    }
                    qsort(cand, (size_t)n, sizeof(cand_t), cand_order);
                    long long keep = n < topk ? n : topk;
                    for (long long slot = 0; slot < topk; ++slot) {
                        long long o = r * topk + slot;
                        if (slot < keep) {
                            out_idx[o] = cand[slot].index;
                            out_score[o] = (float)cand[slot].score + 0.0f;
                            if (out_score64)
                                out_score64[o] = cand[slot].score;
                        } else {
                            out_idx[o] = -1;
                            out_score[o] = -INFINITY;
                            if (out_score64)
                                out_score64[o] = NAN;
                        }
                    }
                    if (out_count)
                        out_count[r] = (int32_t)keep;
                }
            }
            free(qrow);
            free(cand);
        }
    }
    free(keff);
    return status;
}

/* Threads the OpenMP runtime will use (for reporting the CPU baseline). */
int csa_oracle_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
