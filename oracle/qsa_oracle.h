/*
 * CPU oracle for the Qwen Sparse Attention (QSA) layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  This library exists to check the CUDA library
 * against a plain restatement of the method.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it; the product path
 * never calls it and has no CPU fallback.  It shares no code, header or
 * constant with the CUDA library.
 *
 * Everything is single-threaded, fp64, written as loops in the order the
 * method is described:
 *   1. keys are averaged over 4-token micro-blocks           (qo_pool_blocks)
 *   2. a learned indexer scores every complete causal block   (qo_block_scores)
 *   3. the top 512 blocks are kept, lower index wins ties     (qo_select_top_blocks)
 *   4. the attended tokens are those blocks plus the query's
 *      own partial block                                      (qo_attended_tokens)
 *   5. GQA softmax attention over only those tokens           (qo_gqa_attention)
 *
 * Sources: keieiax.jp glossary "Qwen Sparse Attention", section on grouping the
 * context into 4-token micro-blocks (block size 4, an indexer that rates each
 * block, at most 512 blocks = 2,048 tokens per query); blog.cecily.jp/6295, the
 * paragraph summarising Raschka's QSA explainer (keys averaged per block, blocks
 * scored and taken in descending order up to 512) and the trade-off paragraph
 * (budget of 2,048 tokens plus the current remainder).  Readings of points the
 * pages leave open are listed beside each function.
 *
 * bf16 values travel as their 16-bit patterns (uint16_t).
 */
#ifndef QSA_ORACLE_H
#define QSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exact value of a bf16 bit pattern. */
double qo_bf16_value(uint16_t bits);

/* The bf16 nearest to x (ties to even), from the definition of the format:
 * 8 significant bits, fp32's exponent range, gradual underflow, overflow to inf. */
uint16_t qo_round_bf16(double x);

/* Step 1.  pooled[b][:] = bf16( mean_{j<block_size} idx_k[block_size*b + j][:] )
 * for b in [0, n_blocks).  idx_k is [n_blocks*block_size][idx_dim]. */
void qo_pool_blocks(const uint16_t* idx_k, int64_t n_blocks, int32_t idx_dim,
                    int32_t block_size, uint16_t* pooled);

/* Step 2.  scores[b] = sum_h w[h] * max(0, sum_d q_idx[h][d] * pooled[b][d])
 * for the n_cand candidate blocks.  q_idx is [n_idx_heads][idx_dim]. */
void qo_block_scores(const uint16_t* q_idx, const float* w, const uint16_t* pooled,
                     int64_t n_cand, int32_t n_idx_heads, int32_t idx_dim, double* scores);

/* Step 3.  Keep the min(top_k, n_cand) best candidates by (score descending,
 * block index ascending); write them to sel in ascending block order and return
 * the count. */
int32_t qo_select_top_blocks(const double* scores, int64_t n_cand, int32_t top_k, int32_t* sel);

/* Step 4.  Tokens attended by a query at position t: the tokens of the selected
 * blocks, then the query's partial block [block_size*floor((t+1)/block_size), t].
 * Writes ascending token positions and returns how many. */
int64_t qo_attended_tokens(const int32_t* sel, int32_t cnt, int64_t t, int32_t block_size,
                           int64_t* tokens);

/* Step 4, multi-token decode.  keieiax.jp glossary "Qwen Sparse Attention", FAQ on
 * multi-token prediction: the selected top blocks are reused between the
 * speculative steps.  A draft query at position t that reuses the selection made
 * for the query at t_sel (t_sel <= t) attends the tokens of the selected blocks,
 * then every token from the selection query's first incomplete block,
 * block_size*floor((t_sel+1)/block_size), up to t.  With t == t_sel this is
 * qo_attended_tokens.  Writes ascending token positions and returns how many. */
int64_t qo_attended_tokens_shared(const int32_t* sel, int32_t cnt, int64_t t_sel, int64_t t,
                                  int32_t block_size, int64_t* tokens);

/* Step 5.  For each query head h (KV head h / (n_q_heads/n_kv_heads)):
 * out[h][:] = sum_j softmax_j(scale * q[h].k[j]) v[j].
 * q is [n_q_heads][head_dim]; k_rows and v_rows are [n_tok][n_kv_heads][head_dim]. */
void qo_gqa_attention(const uint16_t* q, const uint16_t* k_rows, const uint16_t* v_rows,
                      int64_t n_tok, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                      double scale, double* out);

#ifdef __cplusplus
}
#endif
#endif
