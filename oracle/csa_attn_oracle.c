/*
 * csa_attn_oracle.c -- CPU oracle for the sparse-attention step that consumes
 * the indexer's selection.
 *
 * TEST INFRASTRUCTURE ONLY.  The plain, slow, obviously correct definition
 * that the CUDA sparse-attention kernel is checked against.  Only the tests
 * and the bench's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header, table or helper with the CUDA library (nor with
 * the indexer oracle beside it).
 *
 * What it computes ("StreamIndex: Memory-Bounded Compressed Sparse Attention
 * via Streaming Top-k", abstract: the indexer selects the top-k compressed
 * keys per query and a sparse attention kernel reads only those), in fp64:
 *
 *   for every batch b, query row i and attention head g:
 *     J      = the entries of idx[b,i,0..topk) that are >= 0, in slot order
 *              (the indexer pads unused slots with -1)
 *     z_j    = scale * sum_d qa[b,i,g,d] * kc[b, J_j, d]          (d < Dk)
 *     p_j    = exp(z_j - max_j z_j) / sum_j exp(z_j - max_j z_j)  (softmax over J)
 *     o[b,i,g,e] = sum_j p_j * vc[b, J_j, e]                       (e < Dv)
 *     o = 0 when J is empty.
 *
 * One compressed cache entry per key serves every head (the latent-cache form
 * of multi-head latent attention: keys and values are read from the same
 * per-key rows, shared by all heads).  kc rows are Dk values long; value row
 * s of batch b starts at vc + (b*T + s)*ld_v (ld_v >= Dv), so vc may point
 * into kc's rows (values = a prefix of each key row) or at a separate array.
 * bfloat16 inputs are read as the exact values their bits encode (the upper
 * 16 bits of an IEEE-754 binary32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ATTN_OK 0
#define ATTN_ERR_ARG 1
#define ATTN_ERR_NOMEM 2

static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * rows: n_rows flat query rows r = b*S + i, or NULL for all B*S rows in order.
 * out:  [n_rows, HA, Dv] doubles.
 */
int csa_oracle_sparse_attention(const uint16_t *qa, const uint16_t *kc, const uint16_t *vc,
                                long long ld_v, const int32_t *idx, int B, int S, int T,
                                int HA, int Dk, int Dv, int topk, double scale,
                                const int64_t *rows, long long n_rows, double *out)
{
    if (B < 0 || S < 0 || T < 0 || HA <= 0 || Dk <= 0 || Dv <= 0 || topk <= 0 || ld_v < Dv)
        return ATTN_ERR_ARG;
    if (rows == NULL)
        n_rows = (long long)B * S;
    for (long long r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (long long)B * S)
            return ATTN_ERR_ARG;
    int status = ATTN_OK;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)topk);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)topk);
        if (!z || !sel) {
#pragma omp critical
            status = ATTN_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long long r = 0; r < n_rows; ++r) {
                long long row = rows ? rows[r] : r;
                long long b = row / S;
                /* the selected keys of this query */
                int n = 0;
                for (int j = 0; j < topk; ++j) {
                    int32_t s = idx[row * topk + j];
                    if (s >= 0 && s < T)
                        sel[n++] = s;
                }
                for (int g = 0; g < HA; ++g) {
                    double *o = out + (r * HA + g) * Dv;
                    for (int e = 0; e < Dv; ++e)
                        o[e] = 0.0;
                    if (n == 0)
                        continue;
                    const uint16_t *qg = qa + (row * HA + g) * Dk;
                    double zmax = -INFINITY;
                    for (int j = 0; j < n; ++j) {
                        const uint16_t *kr = kc + (b * T + sel[j]) * (long long)Dk;
                        double dot = 0.0;
                        for (int d = 0; d < Dk; ++d)
                            dot += bf16_value(qg[d]) * bf16_value(kr[d]);
                        z[j] = scale * dot;
                        if (z[j] > zmax)
                            zmax = z[j];
                    }
                    double denom = 0.0;
                    for (int j = 0; j < n; ++j) {
                        z[j] = exp(z[j] - zmax);
                        denom += z[j];
                    }
                    for (int j = 0; j < n; ++j) {
                        const uint16_t *vr = vc + (b * T + sel[j]) * ld_v;
                        double p = z[j] / denom;
                        for (int e = 0; e < Dv; ++e)
                            o[e] += p * bf16_value(vr[e]);
                    }
                }
            }
        }
        free(z);
        free(sel);
    }
    return status;
}
