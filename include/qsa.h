/*
 * qsa.h — C ABI of the B200 (sm_100a) Qwen Sparse Attention (QSA) layer forward.
 *
 * What the layer computes (keieiax.jp glossary "Qwen Sparse Attention", section
 * on grouping the context into 4-token micro-blocks; blog.cecily.jp/6295, the
 * paragraphs summarising Raschka's QSA explainer and the selection budget):
 *
 *   1. indexer keys are averaged over 4-token micro-blocks into a pooled cache,
 *      kept up to date as tokens are appended;
 *   2. a learned indexer scores every complete causal block b of a query at
 *      position t, b < n_c(t) = floor((t+1)/4):
 *          score(b) = sum_h w[h] * ReLU( q_idx[h] . pooled[b] )      (4 heads, dim 64)
 *   3. the 512 best blocks (2,048 tokens) are kept per query, ties going to the
 *      lower block index; the result is a compact ascending index list — no dense
 *      query x key mask ("kq_mask") is ever built;
 *   4. GQA softmax attention runs over the tokens of those blocks plus the
 *      query's own partial block [4*n_c(t), t] (0 to 3 tokens).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller (for example
 *   torch.Tensor.data_ptr()).  The library allocates nothing, keeps no state and
 *   retains no pointer after a call returns.
 * - Every tensor pointer must be 16-byte aligned; tensors are dense, row-major,
 *   with the layouts stated below.  bf16 tensors are IEEE bfloat16.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *   asynchronous; outputs are valid once the stream has synchronised.  Arrays of
 *   lengths, sequence ids and positions live on the device, so a call sequence can
 *   be captured in a CUDA graph.  Host-side integers are upper bounds used only to
 *   size grids and workspaces.
 * - Return value: QSA_OK (0) or a negative QSA_ERR_* code.  Argument errors are
 *   detected on the host before anything is launched.  Errors the host cannot see
 *   (a device-side position outside the cache, a block index outside the bound)
 *   make the kernels skip the offending work and set a bit in the workspace's
 *   device status word (QSA_DEV_*), read with qsa_read_device_status().  No kernel
 *   traps, asserts or waits without bound.
 * - Outputs never alias inputs; `pooled` is the only in-out tensor.
 *
 * Layouts (B = batch, T = kv_capacity, Nb = T/4 pooled blocks, n_q = queries):
 *   q        bf16 [n_q][n_q_heads][head_dim]
 *   k_cache  bf16 [B][n_kv_heads][T][head_dim]   (head-major: one block of one
 *   v_cache  bf16 [B][n_kv_heads][T][head_dim]    head is 1 KiB contiguous)
 *   idx_k    bf16 [B][T][idx_dim]
 *   pooled   bf16 [B][Nb][idx_dim]
 *   q_idx    bf16 [n_q][n_idx_heads][idx_dim]
 *   w        f32  [n_q][n_idx_heads]
 *   q_seq    i32  [n_q]   sequence of each query, in [0, B)
 *   q_pos    i32  [n_q]   0-based position of each query, in [0, T)
 *   sel_idx  i32  [n_q][top_k]  ascending selected blocks, padded with -1
 *   sel_cnt  i32  [n_q]   min(top_k, n_c(t))
 *   out      bf16 [n_q][n_q_heads][head_dim]
 * Query head h reads KV head h / (n_q_heads / n_kv_heads).
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes (return values) ---- */
#define QSA_OK                       0
#define QSA_ERR_INVALID_ARG         -1  /* bad dims, null/misaligned pointer, bad bound */
#define QSA_ERR_WORKSPACE_TOO_SMALL -2  /* ws_bytes < qsa_workspace_bytes(...) */
#define QSA_ERR_UNSUPPORTED         -3  /* valid but not implemented (e.g. head_dim != 128) */
#define QSA_ERR_CUDA                -4  /* a CUDA launch or copy reported an error */

/* ---- device status bits (qsa_read_device_status) ---- */
#define QSA_DEV_BAD_SEQ        0x1u  /* q_seq outside [0, batch): query skipped */
#define QSA_DEV_BAD_POS        0x2u  /* q_pos outside [0, kv_capacity): query skipped */
#define QSA_DEV_BLOCKS_OVER    0x4u  /* n_c(t) > max_blocks: candidates cut at max_blocks */
#define QSA_DEV_BAD_LEN        0x8u  /* len_before/len_after outside [0, kv_capacity] or decreasing */
#define QSA_DEV_BAD_SEL        0x10u /* sel_idx entry outside [0, n_c(t)) or sel_cnt > top_k: skipped */
#define QSA_DEV_TOO_MANY_NEW   0x20u /* len_after - len_before > max_new_tokens: rest not pooled */
#define QSA_DEV_TIMEOUT        0x40u /* a bounded in-kernel wait gave up: results of that call are invalid */

/* ---- forward modes ---- */
#define QSA_MODE_DECODE  0  /* few queries per sequence: split-K attention, multi-CTA select */
#define QSA_MODE_PREFILL 1  /* a chunk of queries of ONE sequence (all q_seq equal) */

typedef struct qsa_dims {
    int32_t batch;        /* B, number of sequences (caches) */
    int32_t n_q_heads;    /* main attention query heads (multiple of n_kv_heads, group <= 16) */
    int32_t n_kv_heads;   /* main attention KV heads */
    int32_t head_dim;     /* must be 128 */
    int32_t n_idx_heads;  /* indexer heads, must be 4 */
    int32_t idx_dim;      /* indexer head dim, must be 64 */
    int32_t block_size;   /* micro-block size, must be 4 */
    int32_t top_k;        /* blocks kept per query, must be 512 */
    int64_t kv_capacity;  /* T, tokens per sequence cache; multiple of 4, < 2^31 */
    float softmax_scale;  /* <= 0 selects 1/sqrt(head_dim) */
} qsa_dims;

/* Workspace bytes qsa_forward needs for n_q queries whose complete causal blocks
 * never exceed max_blocks, in `mode`.  The standalone qsa_topk_blocks and
 * qsa_sparse_attn need at most the QSA_MODE_DECODE figure for the same sizes.
 * Returns 0 on invalid arguments. */
size_t qsa_workspace_bytes(const qsa_dims* dims, int32_t n_q, int64_t max_blocks, int32_t mode);

/* Zero the workspace's status word.  Call once after allocating a workspace. */
int qsa_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream`, copy the device status word (QSA_DEV_* bits, 0 = clean)
 * to *flags and clear it.  Returns QSA_OK or QSA_ERR_CUDA. */
int qsa_read_device_status(void* workspace, uint32_t* flags, void* stream);

/* Human-readable name of a QSA_OK / QSA_ERR_* code (static storage). */
const char* qsa_status_string(int status);

/* Step 1 — micro-block key pooling (4-token means of the indexer keys).
 * For every sequence s, pools each block b completed by the appended range
 * [len_before[s], len_after[s]), i.e. floor(len_before/4) <= b < floor(len_after/4):
 *     pooled[s][b][:] = bf16_rne( 0.25f * (k0 + k1 + k2 + k3) )   (fp32 sum)
 * where k_j = idx_k[s][4b+j][:].  len_before/len_after: device i32 [batch].
 * max_new_tokens: host upper bound on len_after - len_before (grid size).
 * workspace: may be NULL (then device errors are not reported). */
int qsa_pool_block_keys(const qsa_dims* dims, const void* idx_k, void* pooled,
                        const int32_t* len_before, const int32_t* len_after,
                        int32_t max_new_tokens, void* workspace, void* stream);

/* Step 2 — indexer block scores, one row per query:
 *     scores[i][b] = sum_h w[i][h] * ReLU( sum_d q_idx[i][h][d] * pooled[s][b][d] )
 * for b < n_c(q_pos[i]), with bf16 x bf16 products accumulated in fp32, and
 * scores[i][b] = -INFINITY for n_c <= b < max_blocks.  scores is f32 with row
 * stride ld_scores >= max_blocks elements (ld_scores*4 a multiple of 16).
 * workspace: may be NULL (then device errors are not reported). */
int qsa_index_scores(const qsa_dims* dims, const void* q_idx, const float* w, const void* pooled,
                     const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t max_blocks,
                     float* scores, int64_t ld_scores, void* workspace, void* stream);

/* Step 3 — top-k block selection from a score matrix (exact radix select on
 * the fp32 bit patterns, ties to the lower block index).  Candidates of row i
 * are b < n_c(q_pos[i]) (cut at max_blocks).  Writes sel_idx[i][0..cnt) in
 * ascending order, -1 after, and sel_cnt[i] = cnt = min(top_k, n_c).
 * Needs qsa_workspace_bytes(dims, n_q, max_blocks, QSA_MODE_DECODE) bytes. */
int qsa_topk_blocks(const qsa_dims* dims, const float* scores, int64_t ld_scores,
                    const int32_t* q_pos, int32_t n_q, int64_t max_blocks,
                    int32_t* sel_idx, int32_t* sel_cnt, void* workspace, size_t ws_bytes,
                    void* stream);

/* Step 4 — gathered GQA attention over the selected blocks plus the query's
 * partial block:  out[i][h] = sum_j softmax_j(scale * q[i][h].K[s][g][j]) V[s][g][j],
 * g = h / group, j over the 4 tokens of every selected block and the tokens
 * 4*n_c(t) .. t.  fp32 logits, softmax and accumulation; bf16 output (RNE).
 * Needs qsa_workspace_bytes(dims, n_q, 0, QSA_MODE_DECODE) bytes (split-K partials). */
int qsa_sparse_attn(const qsa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                    const int32_t* sel_cnt, int32_t n_q, void* out, void* workspace,
                    size_t ws_bytes, void* stream);

/* Step 4 without a caller workspace.  The pages describe nothing like it: it
 * exists for callers that cannot allocate device memory — an engine whose
 * allocator has already handed all of HBM to its KV cache, a frozen CUDA-graph
 * memory plan, or a plain C host that only owns the tensors it passes — and so
 * cannot provide qsa_sparse_attn's workspace.  Same arguments, layouts, math and
 * results as qsa_sparse_attn, without workspace and ws_bytes.
 * Scratch (split-K partials and completion counters) comes from a 16 MiB array
 * built into the library; every GPU that loads the library holds it until the
 * process exits.  A call takes 4 bytes per (query, KV head) pair for counters
 * plus, when its block lists are split over CTAs (at most 148 pairs), under
 * 2.5 MiB of partials; one needing more than 16 MiB (more than about 4 million
 * pairs) returns QSA_ERR_WORKSPACE_TOO_SMALL before launching.
 * The first call on each device, with that device current, looks the array's
 * device address up (cudaGetSymbolAddress), and so does every later call made
 * outside stream capture (a device reset may move the array); make that first
 * call before any stream capture.  All calls share the array: counters are cleared at the start
 * of each call, and calls whose executions overlap on the GPU race on it.  No
 * device status word: out-of-range indices are skipped but not reported.
 * Nothing in this call allocates memory. */
int qsa_sparse_attn_noalloc(const qsa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                            const int32_t* sel_cnt, int32_t n_q, void* out, void* stream);

/* All inputs of one layer call (see the layouts above). */
typedef struct qsa_forward_args {
    const void* q;            /* bf16 [n_q][n_q_heads][head_dim] */
    const void* k_cache;      /* bf16 [batch][n_kv_heads][kv_capacity][head_dim] */
    const void* v_cache;      /* bf16 [batch][n_kv_heads][kv_capacity][head_dim] */
    const void* idx_k;        /* bf16 [batch][kv_capacity][idx_dim] */
    void* pooled;             /* bf16 [batch][kv_capacity/4][idx_dim], updated in place */
    const void* q_idx;        /* bf16 [n_q][n_idx_heads][idx_dim] */
    const float* w;           /* f32 [n_q][n_idx_heads] */
    const int32_t* len_before;/* i32 [batch] tokens present before this call's append */
    const int32_t* len_after; /* i32 [batch] tokens present after it */
    const int32_t* q_seq;     /* i32 [n_q] */
    const int32_t* q_pos;     /* i32 [n_q] */
    int32_t n_q;              /* number of queries */
    int32_t max_new_tokens;   /* host bound on len_after - len_before */
    int64_t max_blocks;       /* host bound on n_c(q_pos) over all queries */
    int32_t mode;             /* QSA_MODE_DECODE or QSA_MODE_PREFILL */
    int32_t* sel_idx;         /* optional out i32 [n_q][top_k] (NULL: kept in workspace) */
    int32_t* sel_cnt;         /* optional out i32 [n_q] */
    void* out;                /* bf16 [n_q][n_q_heads][head_dim] */
} qsa_forward_args;

/* The whole layer: pool the appended blocks, score, select, attend.
 * Needs qsa_workspace_bytes(dims, n_q, max_blocks, mode) bytes.  Nothing sized
 * n_q x n_keys is ever allocated or built; the library allocates nothing. */
int qsa_forward(const qsa_dims* dims, const qsa_forward_args* args, void* workspace,
                size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* QSA_H */
