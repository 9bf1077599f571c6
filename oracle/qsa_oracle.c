/*
 * CPU oracle for the Qwen Sparse Attention (QSA) layer forward.
 * TEST INFRASTRUCTURE ONLY: see qsa_oracle.h.  Plain C11, fp64, single thread.
 */
#include "qsa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

double qo_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

uint16_t qo_round_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    const int neg = signbit(x) != 0;
    const uint16_t sign = neg ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);

    /* a lies in [2^e, 2^(e+1)); bf16 keeps 8 significant bits, so the spacing of
     * representable values there is 2^(e-7).  Below 2^-126 the spacing stays at
     * the subnormal step 2^-133. */
    int fe;
    frexp(a, &fe);
    int e = fe - 1;
    if (e < -126) e = -126;
    const double step = ldexp(1.0, e - 7);
    const double r = nearbyint(a / step); /* default mode: nearest, ties to even */
    const double y = r * step;
    if (y >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);

    /* y has at most 8 significant bits inside fp32's range: exact as a float,
     * and its low 16 bits are zero. */
    float f = (float)y;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void qo_pool_blocks(const uint16_t* idx_k, int64_t n_blocks, int32_t idx_dim,
                    int32_t block_size, uint16_t* pooled)
{
    for (int64_t b = 0; b < n_blocks; ++b) {
        for (int32_t d = 0; d < idx_dim; ++d) {
            double sum = 0.0;
            for (int32_t j = 0; j < block_size; ++j)
                sum += qo_bf16_value(idx_k[(b * block_size + j) * idx_dim + d]);
            /* the pooled cache stores bf16: round the fp64 mean once */
            pooled[b * idx_dim + d] = qo_round_bf16(sum / (double)block_size);
        }
    }
}

void qo_block_scores(const uint16_t* q_idx, const float* w, const uint16_t* pooled,
                     int64_t n_cand, int32_t n_idx_heads, int32_t idx_dim, double* scores)
{
    for (int64_t b = 0; b < n_cand; ++b) {
        double score = 0.0;
        for (int32_t h = 0; h < n_idx_heads; ++h) {
            double dot = 0.0;
            for (int32_t d = 0; d < idx_dim; ++d)
                dot += qo_bf16_value(q_idx[h * idx_dim + d]) * qo_bf16_value(pooled[b * idx_dim + d]);
            const double relu = dot > 0.0 ? dot : 0.0;
            score += (double)w[h] * relu;
        }
        scores[b] = score;
    }
}

typedef struct {
    double score;
    int32_t block;
} cand_t;

static int by_score_desc_then_block(const void* pa, const void* pb)
{
    const cand_t* a = (const cand_t*)pa;
    const cand_t* b = (const cand_t*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->block > b->block) - (a->block < b->block);
}

static int by_int_asc(const void* pa, const void* pb)
{
    const int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

int32_t qo_select_top_blocks(const double* scores, int64_t n_cand, int32_t top_k, int32_t* sel)
{
    if (n_cand <= 0 || top_k <= 0) return 0;
    cand_t* c = (cand_t*)malloc((size_t)n_cand * sizeof(cand_t));
    if (!c) return -1;
    for (int64_t b = 0; b < n_cand; ++b) {
        c[b].score = scores[b];
        c[b].block = (int32_t)b;
    }
    qsort(c, (size_t)n_cand, sizeof(cand_t), by_score_desc_then_block);
    const int32_t cnt = n_cand < top_k ? (int32_t)n_cand : top_k;
    for (int32_t i = 0; i < cnt; ++i) sel[i] = c[i].block;
    free(c);
    qsort(sel, (size_t)cnt, sizeof(int32_t), by_int_asc);
    return cnt;
}

int64_t qo_attended_tokens(const int32_t* sel, int32_t cnt, int64_t t, int32_t block_size,
                           int64_t* tokens)
{
    int64_t n = 0;
    for (int32_t i = 0; i < cnt; ++i)
        for (int32_t j = 0; j < block_size; ++j)
            tokens[n++] = (int64_t)sel[i] * block_size + j;
    /* the query's own, not yet complete, block: 0 to block_size-1 tokens */
    const int64_t n_complete = (t + 1) / block_size;
    for (int64_t p = n_complete * block_size; p <= t; ++p) tokens[n++] = p;
    return n;
}

int64_t qo_attended_tokens_shared(const int32_t* sel, int32_t cnt, int64_t t_sel, int64_t t,
                                  int32_t block_size, int64_t* tokens)
{
    int64_t n = 0;
    for (int32_t i = 0; i < cnt; ++i)
        for (int32_t j = 0; j < block_size; ++j)
            tokens[n++] = (int64_t)sel[i] * block_size + j;
    /* everything after the complete blocks the selection was made over, up to t */
    const int64_t n_complete_sel = (t_sel + 1) / block_size;
    for (int64_t p = n_complete_sel * block_size; p <= t; ++p) tokens[n++] = p;
    return n;
}

void qo_gqa_attention(const uint16_t* q, const uint16_t* k_rows, const uint16_t* v_rows,
                      int64_t n_tok, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                      double scale, double* out)
{
    const int32_t group = n_q_heads / n_kv_heads;
    double* logit = (double*)malloc((size_t)(n_tok > 0 ? n_tok : 1) * sizeof(double));
    if (!logit) return;
    for (int32_t h = 0; h < n_q_heads; ++h) {
        const int32_t g = h / group;
        double m = -INFINITY;
        for (int64_t j = 0; j < n_tok; ++j) {
            double dot = 0.0;
            for (int32_t d = 0; d < head_dim; ++d)
                dot += qo_bf16_value(q[h * head_dim + d]) *
                       qo_bf16_value(k_rows[(j * n_kv_heads + g) * head_dim + d]);
            logit[j] = scale * dot;
            if (logit[j] > m) m = logit[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < n_tok; ++j) {
            logit[j] = exp(logit[j] - m);
            l += logit[j];
        }
        for (int32_t d = 0; d < head_dim; ++d) {
            double o = 0.0;
            for (int64_t j = 0; j < n_tok; ++j)
                o += logit[j] * qo_bf16_value(v_rows[(j * n_kv_heads + g) * head_dim + d]);
            out[h * head_dim + d] = o / l;
        }
    }
    free(logit);
}
