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
 * Block size and budget: the published setting is 4-token blocks and 512 blocks
 * per query; dims.block_size may be any power of two up to 16 (1 = per-token
 * selection) and dims.top_k any value in [1, QSA_SEL_CAP].  Below, 4 and 512 stand
 * for block_size and top_k, and n_c(t) = floor((t+1)/block_size).
 *
 * Layouts (B = batch, T = kv_capacity, Nb = T/block_size pooled blocks, n_q = queries):
 *   q        bf16 [n_q][n_q_heads][head_dim]
 *   k_cache  bf16 [B][n_kv_heads][T][head_dim]   (head-major: one block of one
 *   v_cache  bf16 [B][n_kv_heads][T][head_dim]    head is 1 KiB contiguous)
 *   idx_k    bf16 [B][T][idx_dim]
 *   pooled   bf16 [B][Nb][idx_dim]
 *   q_idx    bf16 [n_q][n_idx_heads][idx_dim]
 *   w        f32  [n_q][n_idx_heads]
 *   q_seq    i32  [n_q]   sequence of each query, in [0, B)
 *   q_pos    i32  [n_q]   0-based position of each query, in [0, T)
 *   sel_idx  i32  [n_q][QSA_SEL_CAP]  ascending selected blocks, padded with -1
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

/* Capacity of one query's selection: the row stride of every sel_idx array. */
#define QSA_SEL_CAP 512

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
#define QSA_DEV_BAD_PAGE       0x80u /* page-table entry < 0 for an attended token: its block skipped */

/* ---- forward modes ---- */
#define QSA_MODE_DECODE  0  /* few queries per sequence: split-K attention, multi-CTA select */
#define QSA_MODE_PREFILL 1  /* chunks of many queries per sequence (ragged: several sequences per
                                call; keep each sequence's rows contiguous, since every 128-row
                                tile makes one scoring pass per distinct sequence it holds) */
#define QSA_MODE_MIXED   2  /* a serving batch: rows [0, n_decode) decode queries, the rest prefill
                                chunks; one call, one attention launch over every row */

typedef struct qsa_dims {
    int32_t batch;        /* B, number of sequences (caches): 1 .. 65535 */
    int32_t n_q_heads;    /* main attention query heads (multiple of n_kv_heads, group <= 32) */
    int32_t n_kv_heads;   /* main attention KV heads */
    int32_t head_dim;     /* must be 128 */
    int32_t n_idx_heads;  /* indexer heads, must be 4 */
    int32_t idx_dim;      /* indexer head dim, must be 64 */
    int32_t block_size;   /* micro-block size: 1, 2, 4 (published), 8 or 16 */
    int32_t top_k;        /* blocks kept per query: 1 .. QSA_SEL_CAP (512 published) */
    int64_t kv_capacity;  /* T, tokens per sequence cache; multiple of block_size, < 2^31 */
    float softmax_scale;  /* <= 0 selects 1/sqrt(head_dim) */
} qsa_dims;

/* Workspace bytes qsa_forward needs for n_q queries whose complete causal blocks
 * never exceed max_blocks, in `mode` (QSA_MODE_MIXED: any split of n_q into decode
 * and prefill rows).  The standalone qsa_topk_blocks and
 * qsa_sparse_attn need at most the QSA_MODE_DECODE figure for the same sizes.
 * Returns 0 on invalid arguments. */
size_t qsa_workspace_bytes(const qsa_dims* dims, int32_t n_q, int64_t max_blocks, int32_t mode);

/* Zero the whole workspace (its status word and the attention's split counters,
 * which every call leaves at zero again).  Call once after allocating a workspace,
 * before its first use.  One workspace may then serve calls of any entry point and
 * shape in turn (one call at a time), as long as each call's ws_bytes suffices: the
 * counters have the same place in every call's layout, and every other region is
 * written by the call that reads it. */
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

/* Steps 2 and 3 together: scores and the top-k selection of n_q queries, run the
 * way qsa_forward runs them in `mode` (after its pooling step): QSA_MODE_DECODE
 * streams every row's scores through workspace score rows (rows of up to 16,384
 * blocks are selected inside the scoring kernel); QSA_MODE_PREFILL (chunks of
 * queries, ideally contiguous per sequence) scores on the tensor cores and keeps per row only the blocks
 * that can still reach its top 512, so no n_q x n_blocks score matrix exists.
 * Writes sel_idx / sel_cnt as qsa_topk_blocks does.
 * Needs qsa_workspace_bytes(dims, n_q, max_blocks, mode) bytes. */
int qsa_select_blocks(const qsa_dims* dims, const void* q_idx, const float* w, const void* pooled,
                      const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t max_blocks, int32_t mode,
                      int32_t* sel_idx, int32_t* sel_cnt, void* workspace, size_t ws_bytes, void* stream);

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
 * call before any stream capture.  All calls share the array: counters are
 * cleared at the start of each call, and calls whose executions overlap on the
 * GPU race on it.  No
 * device status word: out-of-range indices are skipped but not reported.
 * Nothing in this call allocates memory. */
int qsa_sparse_attn_noalloc(const qsa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                            const int32_t* sel_cnt, int32_t n_q, void* out, void* stream);

/* Step 4, general form: draft queries that share one selection, and paged K/V.
 *
 * Shared selections (keieiax.jp glossary "Qwen Sparse Attention", FAQ on
 * multi-token prediction: the top index is reused between speculative steps):
 * with group_q = k >= 2, queries [k*g, k*g + k) form group g, the k draft tokens
 * of one sequence.  They share selection row g (sel_idx[g], sel_cnt[g], made for
 * the group's first query at t_0 = q_pos[k*g]) and one gather.  Draft query j at
 * position t_j attends the shared blocks plus every token from 4*floor((t_0+1)/4)
 * to t_j.  Requirements (else the query is skipped and QSA_DEV_BAD_SEQ or
 * QSA_DEV_BAD_POS set): same q_seq as the group's first query, and
 * t_0 <= t_j <= 4*floor((t_0+1)/4) + 7 (the tail spans at most two blocks).
 * group_q * (n_q_heads / n_kv_heads) <= 32 and n_q a multiple of group_q.
 * group_q = 1 is qsa_sparse_attn.
 *
 * Paged K/V: with page_table != NULL, k_cache and v_cache are page pools
 * bf16 [n_pages][n_kv_heads][page_tokens][head_dim] and token p of sequence s
 * lies in page page_table[s][p / page_tokens] (i32 [batch][kv_capacity /
 * page_tokens], row p % page_tokens).  page_tokens is a multiple of 4 dividing
 * kv_capacity, so a block never straddles pages.  An attended block whose page
 * entry is outside [0, n_pages) is skipped and QSA_DEV_BAD_PAGE set.  The indexer
 * keys and the pooled cache stay dense per sequence.
 *
 * Workspace: qsa_workspace_bytes(dims, n_q, 0, QSA_MODE_DECODE) bytes. */
typedef struct qsa_attn_args {
    const void* q;              /* bf16 [n_q][n_q_heads][head_dim] */
    const void* k_cache;        /* dense caches or page pools (see above) */
    const void* v_cache;
    const int32_t* q_seq;       /* i32 [n_q] */
    const int32_t* q_pos;       /* i32 [n_q] */
    const int32_t* sel_idx;     /* i32 [n_q / group_q][QSA_SEL_CAP] */
    const int32_t* sel_cnt;     /* i32 [n_q / group_q] */
    int32_t n_q;                /* queries */
    int32_t group_q;            /* queries per shared selection (>= 1) */
    const int32_t* page_table;  /* NULL: dense caches */
    int32_t page_tokens;        /* tokens per page (paged only) */
    int64_t n_pages;            /* pages in each pool (paged only) */
    void* out;                  /* bf16 [n_q][n_q_heads][head_dim] */
} qsa_attn_args;

int qsa_sparse_attn_ex(const qsa_dims* dims, const qsa_attn_args* args, void* workspace, size_t ws_bytes,
                       void* stream);

/* The launch qsa_sparse_attn_ex (and the forward's attention step) makes for n_q
 * queries in groups of group_q: host arithmetic only, no device work, usable for
 * capacity planning.  Few (query group, KV head) pairs split each group's block list
 * over several CTAs; at least 148 pairs take one CTA per pair.  Returns QSA_OK and
 * fills *info, or the argument error qsa_sparse_attn_ex would return.  The cluster
 * merge is reported as the device would run it (0 without a device). */
typedef struct qsa_attn_plan_info {
    int32_t n_split;        /* CTAs per (query group, KV head) */
    int32_t n_stages;       /* K/V stages (64 tokens of K and V each) in flight per CTA */
    int32_t threads;        /* threads per CTA */
    int32_t smem_bytes;     /* dynamic shared memory per CTA */
    int64_t ctas;           /* CTAs of the launch */
    int32_t cluster_merge;  /* 1: the splits merge over distributed shared memory */
    int32_t rows;           /* query-head rows per CTA: group_q x (n_q_heads / n_kv_heads) */
} qsa_attn_plan_info;

int qsa_attn_plan(const qsa_dims* dims, int32_t n_q, int32_t group_q, qsa_attn_plan_info* info);

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
    int32_t* sel_idx;         /* optional out i32 [n_q][QSA_SEL_CAP] (NULL: kept in workspace) */
    int32_t* sel_cnt;         /* optional out i32 [n_q] */
    void* out;                /* bf16 [n_q][n_q_heads][head_dim] */
    /* multi-token decode (QSA_MODE_DECODE only; see qsa_sparse_attn_ex): 0 or 1 =
     * one selection per query; k >= 2: each group of k consecutive draft queries is
     * scored and selected once, for its first query, with q_idx / w / sel_idx /
     * sel_cnt holding one row per group, and attends as qsa_sparse_attn_ex says */
    int32_t group_q;
    /* paged K/V (see qsa_sparse_attn_ex); page_table NULL = dense caches */
    const int32_t* page_table;
    int32_t page_tokens;
    int64_t n_pages;
    /* QSA_MODE_MIXED only: rows [0, n_decode) are decode queries, [n_decode, n_q) prefill
     * chunks (q_idx, w, q_seq, q_pos, sel_idx, sel_cnt, q and out in that row order) */
    int32_t n_decode;
} qsa_forward_args;

/* The whole layer: pool the appended blocks, score, select, attend.
 * Needs qsa_workspace_bytes(dims, n_q, max_blocks, mode) bytes.  Nothing sized
 * n_q x n_keys is ever allocated or built; the library allocates nothing. */
int qsa_forward(const qsa_dims* dims, const qsa_forward_args* args, void* workspace,
                size_t ws_bytes, void* stream);

/* ---- context parallelism: one sequence's blocks spread over several GPUs ----
 *
 * ai-manual.ru, discussion of llama.cpp PR #30965 (closing note): several GPUs add
 * memory but add exchange between the cards.  The layer splits exactly along its two
 * reductions, with two all-gathers between the steps below (made by the caller, e.g.
 * NCCL over NVLink):
 *   1. qsa_cp_select_keys: each GPU scores the blocks it holds and keeps its local
 *      top_k as 64-bit keys (order-preserving score << 32 | ~global block): the
 *      global top_k (score descending, lower block on ties) is a subset of the union;
 *   2. all-gather the keys and counts;
 *   3. qsa_cp_merge_keys: every GPU merges the same union into the same global
 *      selection and keeps the blocks of its own shard;
 *   4. qsa_cp_attn_partial: each GPU attends its selected blocks (and the query's
 *      partial block if the query's last tokens are in its shard) and writes one
 *      unnormalised partial per (query, head);
 *   5. all-gather the partials;  6. qsa_cp_combine: the softmax over the union.
 * A shard is the block range [blk_lo, blk_lo + n_local) of every sequence, held in
 * the usual layouts with kv_capacity = n_local * block_size tokens (so `shard`
 * describes the local caches); positions (q_pos) stay global.  Decode-shaped calls
 * (few queries per sequence).  Keys: u64 [n_q][QSA_SEL_CAP] (unused slots 0),
 * counts i32 [n_q]; gathered arrays are rank-major ([n_ranks][n_q]...).  Partials:
 * f32 [n_q][n_q_heads][132] = (max, sum, 2 unused, 128 weighted values), exp2 domain.
 * Workspace: qsa_cp_workspace_bytes(shard, n_q), initialised with qsa_workspace_init. */
size_t qsa_cp_workspace_bytes(const qsa_dims* shard, int32_t n_q);
int qsa_cp_select_keys(const qsa_dims* shard, const void* q_idx, const float* w, const void* pooled_shard,
                       const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t blk_lo, uint64_t* keys,
                       int32_t* key_cnt, void* workspace, size_t ws_bytes, void* stream);
/* n_ranks <= 8.  sel_local / cnt_local: this shard's blocks of the global selection,
 * ascending, as shard-local indices (-1 padded); sel_global / cnt_global (optional,
 * NULL to skip): the whole global selection. */
int qsa_cp_merge_keys(const qsa_dims* shard, int32_t n_ranks, const uint64_t* keys_all, const int32_t* cnt_all,
                      int32_t n_q, int64_t blk_lo, int32_t* sel_local, int32_t* cnt_local, int32_t* sel_global,
                      int32_t* cnt_global, void* stream);
int qsa_cp_attn_partial(const qsa_dims* shard, const void* q, const void* k_shard, const void* v_shard,
                        const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t blk_lo,
                        const int32_t* sel_local, const int32_t* cnt_local, float* part, void* workspace,
                        size_t ws_bytes, void* stream);
int qsa_cp_combine(const qsa_dims* dims, int32_t n_ranks, const float* parts_all, int32_t n_q, void* out,
                   void* stream);

#ifdef __cplusplus
}
#endif
#endif /* QSA_H */
