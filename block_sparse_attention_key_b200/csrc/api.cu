// Host entry points of libqsa.so: argument checks, workspace layout, launch order.
// The C ABI itself is documented in include/qsa.h.

#include <cmath>
#include <cstdint>

#include "qsa_internal.cuh"

namespace qsa {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

}  // namespace

// Argument checks shared by every entry point (declared in qsa_internal.cuh).
bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

int check_dims(const qsa_dims* d)
{
    if (!d) return QSA_ERR_INVALID_ARG;
    if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1) return QSA_ERR_INVALID_ARG;
    if (d->n_q_heads % d->n_kv_heads != 0) return QSA_ERR_INVALID_ARG;
    // block size: a power of two up to 16 (4 in the published setting, 1 for per-token
    // selection); top_k: 1 .. 512 blocks (512 published)
    if (d->block_size < 1 || d->block_size > kMaxBlockSize || (d->block_size & (d->block_size - 1)) != 0)
        return QSA_ERR_INVALID_ARG;
    if (d->top_k < 1 || d->top_k > kSelCap) return QSA_ERR_INVALID_ARG;
    if (d->kv_capacity <= 0 || d->kv_capacity % d->block_size != 0 || d->kv_capacity >= (1ll << 31))
        return QSA_ERR_INVALID_ARG;
    if (!std::isfinite(d->softmax_scale)) return QSA_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim || d->n_idx_heads != kIdxHeads || d->idx_dim != kIdxDim)
        return QSA_ERR_UNSUPPORTED;
    if (d->n_q_heads / d->n_kv_heads > kMaxGroup) return QSA_ERR_UNSUPPORTED;
    if (d->batch > 65535) return QSA_ERR_UNSUPPORTED;  // sequences index a grid dimension of the pooling launch
    return QSA_OK;
}

int check_rows(const qsa_dims* d, int32_t n_q, int64_t max_blocks)
{
    if (n_q < 0 || max_blocks < 0 || max_blocks > d->kv_capacity / d->block_size) return QSA_ERR_INVALID_ARG;
    if (n_q > 65535) return QSA_ERR_UNSUPPORTED;
    return QSA_OK;
}

int check_groups(const qsa_dims* d, int32_t n_q, int32_t group_q)
{
    if (group_q < 1 || n_q % group_q != 0) return QSA_ERR_INVALID_ARG;
    if ((int64_t)group_q * (d->n_q_heads / d->n_kv_heads) > 32) return QSA_ERR_UNSUPPORTED;
    return QSA_OK;
}

int check_pages(const qsa_dims* d, const int32_t* page_table, int32_t page_tokens, int64_t n_pages)
{
    if (!page_table) return QSA_OK;
    if (!aligned16(page_table) || page_tokens < 1 || page_tokens % d->block_size != 0 ||
        d->kv_capacity % page_tokens != 0 || n_pages < 1 || n_pages > (1ll << 31) - 1)
        return QSA_ERR_INVALID_ARG;
    return QSA_OK;
}

int select_chunk(int64_t max_blocks, int32_t n_rows)
{
    if (max_blocks <= 0) return 256;
    const int64_t rows = n_rows > 0 ? n_rows : 1;
    // one wave at two CTAs per SM on the 148 SMs of a B200: each CTA streams a long
    // run of blocks with its copies in flight instead of paying set-up per short chunk
    int64_t c = (max_blocks * rows + 295) / 296;
    c = (c + 255) / 256 * 256;
    const int64_t cap = (max_blocks + 255) / 256 * 256;
    if (c > cap) c = cap;
    if (c > 16384) c = 16384;
    if (c < 256) c = 256;
    return (int)c;
}

WsLayout plan_workspace(const qsa_dims& d, int32_t n_q, int64_t max_blocks, int32_t mode)
{
    WsLayout L;
    size_t off = kAlign;  // status word
    // decode rows go through the score-row select; prefill chunks through the tensor-core path
    const int32_t rows = (max_blocks > 0 && mode == QSA_MODE_DECODE) ? n_q : 0;
    L.score_rows = rows;
    L.chunk = select_chunk(max_blocks, rows);
    L.n_chunks = max_blocks > 0 ? (int)((max_blocks + L.chunk - 1) / L.chunk) : 0;

    // zeroed region: attention split counters, then the select control blocks.  The
    // counters' region has one size in every layout, so calls of any shape that share
    // a workspace find only counters there (each left at zero by its last split)
    L.attn_cnt = off;
    L.ctrl = off + align_up(attn_counter_bytes());
    L.ctrl_bytes = (L.ctrl - L.attn_cnt) + (size_t)rows * sizeof(TopkCtrl);
    off = L.attn_cnt + align_up(L.ctrl_bytes);
    L.cand = off;
    off += align_up((size_t)rows * kCandCap * 8);
    L.tmp = off;
    off += align_up((size_t)rows * kSelCap * 4);
    L.score_ld = (max_blocks + 3) / 4 * 4;
    L.scores = off;
    off += align_up((size_t)rows * L.score_ld * 4);
    L.sel = off;
    off += align_up((size_t)n_q * kSelCap * 4 + (size_t)n_q * 4);
    // decode attention partials, for a merge of split CTAs through global memory
    L.partial = off;
    if (n_q > 0) off += align_up(attn_partial_bytes());
    if (mode == QSA_MODE_PREFILL && max_blocks > 0 && n_q > 0) {
        L.pf_split = prefill_splits(n_q, max_blocks);
        const size_t segs = (size_t)n_q * prefill_segments(L.pf_split);
        L.pf_cand = off;
        off += align_up(segs * prefill_seg_cap() * 8);
        L.pf_cnt = off;
        off += align_up(segs * 4);
        // thresholds, then the worklist count: zeroed together
        L.pf_theta = off;
        L.pf_work = off + (size_t)n_q * 4;
        off += align_up((size_t)(2 * n_q + 1) * 4);
        L.pf_shist = off;
        off += align_up((size_t)n_q * prefill_shist_words(L.pf_split) * 4);
        L.pf_fb_ctas = n_q < 64 ? n_q : 64;
        L.pf_scratch = off;
        off += align_up((size_t)L.pf_fb_ctas * max_blocks * 4);
    }
    L.qpos_loc = off;
    off += align_up((size_t)n_q * 4);
    L.total = off;
    return L;
}

// Gathered attention for one call (k_sparse_attn): few (query group, KV head) pairs
// split their block lists over the SMs, many pairs run one CTA per pair.
static cudaError_t run_attention(const qsa_dims& d, const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx,
                                 const int32_t* sel_cnt, const int32_t* page_table, int32_t page_tokens,
                                 int64_t n_pages, int32_t n_q, int32_t group_q, void* out, const WsLayout& L,
                                 char* ws, cudaStream_t st, bool pdl, bool counters_zeroed)
{
    const int64_t n_groups = n_q / group_q;
    float* partial = (float*)(ws + L.partial);
    unsigned* counters = (unsigned*)(ws + L.attn_cnt);
    return launch_sparse_attn(d, q, k_cache, v_cache, q_seq, q_pos, sel_idx, sel_cnt, page_table, page_tokens,
                              n_pages, n_groups, group_q, out, partial, counters, (unsigned*)ws, st, pdl, true,
                              counters_zeroed);
}

// Steps 2 + 3 for `n_rows` selection rows (one per group of group_q queries) into
// sel_idx / sel_cnt.  Decode rows expect their control blocks zeroed already.
static cudaError_t run_select(const qsa_dims& d, const void* q_idx, const float* w, const void* pooled,
                              const int32_t* q_seq, const int32_t* q_pos, int32_t n_rows, int32_t group_q,
                              int64_t max_blocks, int32_t mode, int32_t* sel_idx, int32_t* sel_cnt,
                              const WsLayout& L, char* ws, unsigned* status, cudaStream_t st, bool pdl)
{
    cudaError_t e = cudaSuccess;
    if (max_blocks == 0) {
        e = cudaMemsetAsync(sel_idx, 0xFF, (size_t)n_rows * kSelCap * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(sel_cnt, 0, (size_t)n_rows * 4, st);
        return e;
    }
    if (mode == QSA_MODE_DECODE) {
        TopkCtrl* ctrl = (TopkCtrl*)(ws + L.ctrl);
        float* scores = (float*)(ws + L.scores);
        // rows of up to 16,384 blocks are selected by the scoring kernel's last CTA per row
        const bool in_kernel = max_blocks <= kScoreFinishMaxBlocks;
        e = launch_score_decode(d, q_idx, w, pooled, q_seq, q_pos, 0, n_rows, max_blocks, scores, L.score_ld,
                                L.chunk, ctrl, in_kernel ? sel_idx : nullptr, in_kernel ? sel_cnt : nullptr, status,
                                st, pdl, group_q);
        if (e != cudaSuccess || in_kernel) return e;
        return launch_topk(scores, L.score_ld, q_pos, 0, n_rows, max_blocks, d.kv_capacity, d.block_size, d.top_k,
                           L.chunk, L.n_chunks, ctrl, (unsigned long long*)(ws + L.cand), (int32_t*)(ws + L.tmp), sel_idx, sel_cnt, true,
                           status, st, pdl);
    }
    // prefill chunk: tensor-core scoring with streaming admission.  The rows' thresholds
    // and the fallback worklist's count start at zero; the count sits after the
    // thresholds of the layout's n_q rows, which a mixed call's n_rows may be fewer than
    e = cudaMemsetAsync(ws + L.pf_theta, 0, L.pf_work + 4 - L.pf_theta, st);
    if (e != cudaSuccess) return e;
    return launch_prefill_select(d, q_idx, w, pooled, q_seq, q_pos, n_rows, max_blocks, L.pf_split,
                                 (unsigned long long*)(ws + L.pf_cand), (unsigned*)(ws + L.pf_cnt),
                                 (unsigned*)(ws + L.pf_theta), (uint32_t*)(ws + L.pf_shist),
                                 (int32_t*)(ws + L.pf_work), (float*)(ws + L.pf_scratch), L.pf_fb_ctas, sel_idx,
                                 sel_cnt, status, st);
}

// A serving batch in one call: rows [0, n_decode) are decode queries (any sequences,
// scored through score rows), rows [n_decode, n_q) are prefill chunks (tensor-core
// scoring); one pooling launch before and one attention launch over every row after.
// The workspace holds a decode layout, then a prefill layout; the status word is the
// first one's.
static int forward_mixed(const qsa_dims& d, const qsa_forward_args& a, char* ws, size_t ws_bytes, cudaStream_t st)
{
    const int32_t n_q = a.n_q, n_dec = a.n_decode, n_pf = n_q - n_dec;
    const WsLayout Ld = plan_workspace(d, n_q, a.max_blocks, QSA_MODE_DECODE);
    const WsLayout Lp = plan_workspace(d, n_q, a.max_blocks, QSA_MODE_PREFILL);
    if (ws_bytes < Ld.total + Lp.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    unsigned* status = (unsigned*)ws;
    int32_t* sel_idx = a.sel_idx ? a.sel_idx : (int32_t*)(ws + Ld.sel);
    int32_t* sel_cnt = a.sel_cnt ? a.sel_cnt : (int32_t*)(ws + Ld.sel) + (size_t)n_q * kSelCap;
    // pool the appended blocks; the same launch clears the decode rows' control blocks
    cudaError_t e = launch_pool(d, a.idx_k, a.pooled, a.len_before, a.len_after, a.max_new_tokens, ws + Ld.attn_cnt,
                                Ld.ctrl_bytes, status, st);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    if (n_dec > 0) {
        e = run_select(d, a.q_idx, a.w, a.pooled, a.q_seq, a.q_pos, n_dec, 1, a.max_blocks, QSA_MODE_DECODE, sel_idx,
                       sel_cnt, Ld, ws, status, st, false);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    if (n_pf > 0) {
        const size_t qrow = (size_t)kIdxHeads * kIdxDim * 2;
        e = run_select(d, (const char*)a.q_idx + (size_t)n_dec * qrow, a.w + (size_t)n_dec * kIdxHeads, a.pooled,
                       a.q_seq + n_dec, a.q_pos + n_dec, n_pf, 1, a.max_blocks, QSA_MODE_PREFILL,
                       sel_idx + (size_t)n_dec * kSelCap, sel_cnt + n_dec, Lp, ws + Ld.total, status, st, false);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    if (n_q == 0) return QSA_OK;
    return cuda_status(run_attention(d, a.q, a.k_cache, a.v_cache, a.q_seq, a.q_pos, sel_idx, sel_cnt, a.page_table,
                                     a.page_tokens, a.n_pages, n_q, 1, a.out, Ld, ws, st, false, true));
}

}  // namespace qsa

using namespace qsa;

extern "C" {

size_t qsa_workspace_bytes(const qsa_dims* dims, int32_t n_q, int64_t max_blocks, int32_t mode)
{
    if (check_dims(dims) != QSA_OK || check_rows(dims, n_q, max_blocks) != QSA_OK) return 0;
    if (mode == QSA_MODE_MIXED)
        return plan_workspace(*dims, n_q, max_blocks, QSA_MODE_DECODE).total +
               plan_workspace(*dims, n_q, max_blocks, QSA_MODE_PREFILL).total;
    if (mode != QSA_MODE_DECODE && mode != QSA_MODE_PREFILL) return 0;
    return plan_workspace(*dims, n_q, max_blocks, mode).total;
}

int qsa_workspace_init(void* workspace, size_t ws_bytes, void* stream)
{
    if (!aligned16(workspace) || ws_bytes < kAlign) return QSA_ERR_INVALID_ARG;
    // the status word and every completion counter start at zero (counters return to
    // zero at the end of every launch that uses them)
    return cuda_status(cudaMemsetAsync(workspace, 0, ws_bytes, (cudaStream_t)stream));
}

int qsa_read_device_status(void* workspace, uint32_t* flags, void* stream)
{
    if (!aligned16(workspace) || !flags) return QSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof h, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof h, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    *flags = h;
    return QSA_OK;
}

const char* qsa_status_string(int status)
{
    switch (status) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_WORKSPACE_TOO_SMALL: return "QSA_ERR_WORKSPACE_TOO_SMALL";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
    default: return "QSA_ERR_UNKNOWN";
    }
}

int qsa_pool_block_keys(const qsa_dims* dims, const void* idx_k, void* pooled, const int32_t* len_before,
                        const int32_t* len_after, int32_t max_new_tokens, void* workspace, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if (!aligned16(idx_k) || !aligned16(pooled) || !aligned16(len_before) || !aligned16(len_after))
        return QSA_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return QSA_ERR_INVALID_ARG;
    if (max_new_tokens < 0 || (int64_t)max_new_tokens > dims->kv_capacity) return QSA_ERR_INVALID_ARG;
    if (max_new_tokens == 0) return QSA_OK;
    return cuda_status(launch_pool(*dims, idx_k, pooled, len_before, len_after, max_new_tokens, nullptr, 0,
                                   (unsigned*)workspace, (cudaStream_t)stream));
}

int qsa_index_scores(const qsa_dims* dims, const void* q_idx, const float* w, const void* pooled,
                     const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t max_blocks,
                     float* scores, int64_t ld_scores, void* workspace, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(dims, n_q, max_blocks)) != QSA_OK) return rc;
    if (n_q == 0 || max_blocks == 0) return QSA_OK;
    if (!aligned16(q_idx) || !aligned16(w) || !aligned16(pooled) || !aligned16(q_seq) || !aligned16(q_pos) ||
        !aligned16(scores))
        return QSA_ERR_INVALID_ARG;
    if (workspace && !aligned16(workspace)) return QSA_ERR_INVALID_ARG;
    if (ld_scores < max_blocks || ld_scores % 4 != 0) return QSA_ERR_INVALID_ARG;
    const int chunk = select_chunk(max_blocks, n_q);
    return cuda_status(launch_score_decode(*dims, q_idx, w, pooled, q_seq, q_pos, 0, n_q, max_blocks, scores,
                                           ld_scores, chunk, nullptr, nullptr, nullptr, (unsigned*)workspace,
                                           (cudaStream_t)stream));
}

int qsa_topk_blocks(const qsa_dims* dims, const float* scores, int64_t ld_scores, const int32_t* q_pos,
                    int32_t n_q, int64_t max_blocks, int32_t* sel_idx, int32_t* sel_cnt, void* workspace,
                    size_t ws_bytes, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(dims, n_q, max_blocks)) != QSA_OK) return rc;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(q_pos) || !aligned16(sel_idx) || !aligned16(sel_cnt) || !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    if (max_blocks > 0 && (!aligned16(scores) || ld_scores < max_blocks)) return QSA_ERR_INVALID_ARG;
    const WsLayout L = plan_workspace(*dims, n_q, max_blocks, QSA_MODE_DECODE);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    if (max_blocks == 0) {
        // no candidates at all: empty selections
        cudaError_t e = cudaMemsetAsync(sel_idx, 0xFF, (size_t)n_q * kSelCap * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(sel_cnt, 0, (size_t)n_q * 4, st);
        return cuda_status(e);
    }
    cudaError_t e = cudaMemsetAsync(ws + L.attn_cnt, 0, L.ctrl_bytes, st);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    return cuda_status(launch_topk(scores, ld_scores, q_pos, 0, n_q, max_blocks, dims->kv_capacity,
                                   dims->block_size, dims->top_k, L.chunk, L.n_chunks, (TopkCtrl*)(ws + L.ctrl), (unsigned long long*)(ws + L.cand),
                                   (int32_t*)(ws + L.tmp), sel_idx, sel_cnt, false, (unsigned*)ws, st));
}

int qsa_sparse_attn(const qsa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx, const int32_t* sel_cnt,
                    int32_t n_q, void* out, void* workspace, size_t ws_bytes, void* stream)
{
    qsa_attn_args a = {};
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.q_seq = q_seq;
    a.q_pos = q_pos;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.n_q = n_q;
    a.group_q = 1;
    a.out = out;
    return qsa_sparse_attn_ex(dims, &a, workspace, ws_bytes, stream);
}

int qsa_sparse_attn_ex(const qsa_dims* dims, const qsa_attn_args* a, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if (!a) return QSA_ERR_INVALID_ARG;
    if ((rc = check_rows(dims, a->n_q, 0)) != QSA_OK) return rc;
    if ((rc = check_groups(dims, a->n_q, a->group_q < 1 ? 0 : a->group_q)) != QSA_OK) return rc;
    if ((rc = check_pages(dims, a->page_table, a->page_tokens, a->n_pages)) != QSA_OK) return rc;
    if (a->n_q == 0) return QSA_OK;
    if (!aligned16(a->q) || !aligned16(a->k_cache) || !aligned16(a->v_cache) || !aligned16(a->q_seq) ||
        !aligned16(a->q_pos) || !aligned16(a->sel_idx) || !aligned16(a->sel_cnt) || !aligned16(a->out) ||
        !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    const WsLayout L = plan_workspace(*dims, a->n_q, 0, QSA_MODE_DECODE);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    // split counters: zero since qsa_workspace_init, and every merge resets its own
    return cuda_status(run_attention(*dims, a->q, a->k_cache, a->v_cache, a->q_seq, a->q_pos, a->sel_idx, a->sel_cnt,
                                     a->page_table, a->page_tokens, a->n_pages, a->n_q, a->group_q, a->out, L,
                                     (char*)workspace, (cudaStream_t)stream, false, true));
}

int qsa_attn_plan(const qsa_dims* dims, int32_t n_q, int32_t group_q, qsa_attn_plan_info* info)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if (!info) return QSA_ERR_INVALID_ARG;
    if ((rc = check_rows(dims, n_q, 0)) != QSA_OK) return rc;
    if ((rc = check_groups(dims, n_q, group_q < 1 ? 0 : group_q)) != QSA_OK) return rc;
    *info = qsa_attn_plan_info{};
    if (n_q == 0) return QSA_OK;
    int n_split = 0, stages = 0, threads = 0, smem = 0, cluster = 0, rows = 0;
    int64_t ctas = 0;
    if (!describe_sparse_attn(*dims, n_q / group_q, group_q, true, &n_split, &stages, &threads, &smem, &ctas, &cluster,
                              &rows))
        return QSA_ERR_UNSUPPORTED;
    info->n_split = n_split;
    info->n_stages = stages;
    info->threads = threads;
    info->smem_bytes = smem;
    info->ctas = ctas;
    info->cluster_merge = cluster;
    info->rows = rows;
    return QSA_OK;
}

int qsa_select_blocks(const qsa_dims* dims, const void* q_idx, const float* w, const void* pooled,
                      const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t max_blocks, int32_t mode,
                      int32_t* sel_idx, int32_t* sel_cnt, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(dims, n_q, max_blocks)) != QSA_OK) return rc;
    if (mode != QSA_MODE_DECODE && mode != QSA_MODE_PREFILL) return QSA_ERR_INVALID_ARG;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(q_idx) || !aligned16(w) || !aligned16(pooled) || !aligned16(q_seq) || !aligned16(q_pos) ||
        !aligned16(sel_idx) || !aligned16(sel_cnt) || !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    const WsLayout L = plan_workspace(*dims, n_q, max_blocks, mode);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    if (mode == QSA_MODE_DECODE && max_blocks > 0) {
        const cudaError_t e = cudaMemsetAsync(ws + L.ctrl, 0, (size_t)n_q * sizeof(TopkCtrl), st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    return cuda_status(run_select(*dims, q_idx, w, pooled, q_seq, q_pos, n_q, 1, max_blocks, mode, sel_idx, sel_cnt,
                                  L, ws, (unsigned*)ws, st, false));
}

int qsa_forward(const qsa_dims* dims, const qsa_forward_args* a, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if (!a) return QSA_ERR_INVALID_ARG;
    if ((rc = check_rows(dims, a->n_q, a->max_blocks)) != QSA_OK) return rc;
    if (a->mode != QSA_MODE_DECODE && a->mode != QSA_MODE_PREFILL && a->mode != QSA_MODE_MIXED)
        return QSA_ERR_INVALID_ARG;
    if (a->mode == QSA_MODE_MIXED && (a->n_decode < 0 || a->n_decode > a->n_q)) return QSA_ERR_INVALID_ARG;
    const int32_t group_q = a->group_q < 1 ? 1 : a->group_q;
    if (group_q > 1 && a->mode != QSA_MODE_DECODE) return QSA_ERR_INVALID_ARG;
    if ((rc = check_groups(dims, a->n_q, group_q)) != QSA_OK) return rc;
    if ((rc = check_pages(dims, a->page_table, a->page_tokens, a->n_pages)) != QSA_OK) return rc;
    if (a->max_new_tokens < 0 || (int64_t)a->max_new_tokens > dims->kv_capacity) return QSA_ERR_INVALID_ARG;
    if (!aligned16(a->idx_k) || !aligned16(a->pooled) || !aligned16(a->len_before) || !aligned16(a->len_after) ||
        !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    if (a->n_q > 0 && (!aligned16(a->q) || !aligned16(a->k_cache) || !aligned16(a->v_cache) ||
                       !aligned16(a->q_idx) || !aligned16(a->w) || !aligned16(a->q_seq) ||
                       !aligned16(a->q_pos) || !aligned16(a->out)))
        return QSA_ERR_INVALID_ARG;
    if ((a->sel_idx && !aligned16(a->sel_idx)) || (a->sel_cnt && !aligned16(a->sel_cnt)))
        return QSA_ERR_INVALID_ARG;
    const int32_t n_q = a->n_q;
    const int32_t n_groups = n_q / group_q;  // selection rows
    if (a->mode == QSA_MODE_MIXED) return forward_mixed(*dims, *a, (char*)workspace, ws_bytes, (cudaStream_t)stream);
    const WsLayout L = plan_workspace(*dims, n_q, a->max_blocks, a->mode);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    unsigned* status = (unsigned*)ws;
    cudaError_t e = cudaSuccess;
    int32_t* sel_idx = a->sel_idx ? a->sel_idx : (int32_t*)(ws + L.sel);
    int32_t* sel_cnt = a->sel_cnt ? a->sel_cnt : (int32_t*)(ws + L.sel) + (size_t)n_q * kSelCap;
    if (n_q > 0 && a->max_blocks > 0 && a->mode == QSA_MODE_DECODE) {
        // decode chain, each kernel launched as a programmatic dependent of the one
        // before: pool (+ clearing of the split counters and select control blocks),
        // scores with the digit-1 histogram, select, attention; one selection row per
        // group of draft queries, scored at the group's first query
        e = launch_pool(*dims, a->idx_k, a->pooled, a->len_before, a->len_after, a->max_new_tokens, ws + L.attn_cnt,
                        L.ctrl_bytes, status, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
        e = run_select(*dims, a->q_idx, a->w, a->pooled, a->q_seq, a->q_pos, n_groups, group_q, a->max_blocks,
                       QSA_MODE_DECODE, sel_idx, sel_cnt, L, ws, status, st, true);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
        return cuda_status(run_attention(*dims, a->q, a->k_cache, a->v_cache, a->q_seq, a->q_pos, sel_idx, sel_cnt,
                                         a->page_table, a->page_tokens, a->n_pages, n_q, group_q, a->out, L, ws, st,
                                         true, true));
    }

    if (a->max_new_tokens > 0) {
        e = launch_pool(*dims, a->idx_k, a->pooled, a->len_before, a->len_after, a->max_new_tokens, nullptr, 0,
                        status, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    if (n_q == 0) return QSA_OK;

    // a prefill chunk (or a decode call with no complete block anywhere)
    e = run_select(*dims, a->q_idx, a->w, a->pooled, a->q_seq, a->q_pos, n_groups, group_q, a->max_blocks,
                   QSA_MODE_PREFILL, sel_idx, sel_cnt, L, ws, status, st, false);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    return cuda_status(run_attention(*dims, a->q, a->k_cache, a->v_cache, a->q_seq, a->q_pos, sel_idx, sel_cnt,
                                     a->page_table, a->page_tokens, a->n_pages, n_q, group_q, a->out, L, ws, st, false,
                                     true));
}

// ---------------------------------------------------------------- context parallelism

static int check_shard(const qsa_dims* shard, int32_t n_q, int64_t blk_lo)
{
    int rc = check_dims(shard);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(shard, n_q, 0)) != QSA_OK) return rc;
    if (blk_lo < 0 || (blk_lo + shard->kv_capacity / shard->block_size) * shard->block_size >= (1ll << 31))
        return QSA_ERR_INVALID_ARG;
    return QSA_OK;
}

size_t qsa_cp_workspace_bytes(const qsa_dims* shard, int32_t n_q)
{
    if (check_shard(shard, n_q, 0) != QSA_OK) return 0;
    return plan_workspace(*shard, n_q, shard->kv_capacity / shard->block_size, QSA_MODE_DECODE).total;
}

int qsa_cp_select_keys(const qsa_dims* shard, const void* q_idx, const float* w, const void* pooled_shard,
                       const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t blk_lo, uint64_t* keys,
                       int32_t* key_cnt, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_shard(shard, n_q, blk_lo);
    if (rc != QSA_OK) return rc;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(q_idx) || !aligned16(w) || !aligned16(pooled_shard) || !aligned16(q_seq) || !aligned16(q_pos) ||
        !aligned16(keys) || !aligned16(key_cnt) || !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    const int64_t n_local = shard->kv_capacity / shard->block_size;
    const WsLayout L = plan_workspace(*shard, n_q, n_local, QSA_MODE_DECODE);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    int32_t* pos_loc = (int32_t*)(ws + L.qpos_loc);
    int32_t* sel = (int32_t*)(ws + L.sel);
    int32_t* cnt = sel + (size_t)n_q * kSelCap;
    // positions outside the shard are expected here: their flags go to a word nobody reads
    unsigned* quiet = (unsigned*)ws + 1;
    cudaError_t e = launch_cp_local_pos(q_pos, n_q, blk_lo * shard->block_size, shard->kv_capacity, pos_loc, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws + L.ctrl, 0, (size_t)n_q * sizeof(TopkCtrl), st);
    if (e == cudaSuccess)
        e = run_select(*shard, q_idx, w, pooled_shard, q_seq, pos_loc, n_q, 1, n_local, QSA_MODE_DECODE, sel, cnt, L, ws,
                       quiet, st, false);
    if (e == cudaSuccess)
        e = launch_cp_keys((const float*)(ws + L.scores), L.score_ld, sel, cnt, n_q, blk_lo,
                           (unsigned long long*)keys, key_cnt, st);
    return cuda_status(e);
}

int qsa_cp_merge_keys(const qsa_dims* shard, int32_t n_ranks, const uint64_t* keys_all, const int32_t* cnt_all,
                      int32_t n_q, int64_t blk_lo, int32_t* sel_local, int32_t* cnt_local, int32_t* sel_global,
                      int32_t* cnt_global, void* stream)
{
    int rc = check_shard(shard, n_q, blk_lo);
    if (rc != QSA_OK) return rc;
    if (n_ranks < 1 || n_ranks > kCandCap / kSelCap) return QSA_ERR_UNSUPPORTED;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(keys_all) || !aligned16(cnt_all) || !aligned16(sel_local) || !aligned16(cnt_local) ||
        (sel_global && !aligned16(sel_global)) || (cnt_global && !aligned16(cnt_global)))
        return QSA_ERR_INVALID_ARG;
    return cuda_status(launch_cp_merge((const unsigned long long*)keys_all, cnt_all, n_ranks, n_q, shard->top_k,
                                       blk_lo, shard->kv_capacity / shard->block_size, sel_local, cnt_local,
                                       sel_global, cnt_global, (cudaStream_t)stream));
}

int qsa_cp_attn_partial(const qsa_dims* shard, const void* q, const void* k_shard, const void* v_shard,
                        const int32_t* q_seq, const int32_t* q_pos, int32_t n_q, int64_t blk_lo,
                        const int32_t* sel_local, const int32_t* cnt_local, float* part, void* workspace,
                        size_t ws_bytes, void* stream)
{
    int rc = check_shard(shard, n_q, blk_lo);
    if (rc != QSA_OK) return rc;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(q) || !aligned16(k_shard) || !aligned16(v_shard) || !aligned16(q_seq) || !aligned16(q_pos) ||
        !aligned16(sel_local) || !aligned16(cnt_local) || !aligned16(part) || !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    const WsLayout L = plan_workspace(*shard, n_q, shard->kv_capacity / shard->block_size, QSA_MODE_DECODE);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    int32_t* pos_loc = (int32_t*)(ws + L.qpos_loc);
    unsigned* quiet = (unsigned*)ws + 1;
    cudaError_t e = launch_cp_local_pos(q_pos, n_q, blk_lo * shard->block_size, shard->kv_capacity, pos_loc, st);
    if (e == cudaSuccess)
        e = launch_sparse_attn(*shard, q, k_shard, v_shard, q_seq, pos_loc, sel_local, cnt_local, nullptr, 0, 0, n_q,
                               1, nullptr, (float*)(ws + L.partial), (unsigned*)(ws + L.attn_cnt), quiet, st, false,
                               true, true, part);
    return cuda_status(e);
}

int qsa_cp_combine(const qsa_dims* dims, int32_t n_ranks, const float* parts_all, int32_t n_q, void* out, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(dims, n_q, 0)) != QSA_OK) return rc;
    if (n_ranks < 1) return QSA_ERR_INVALID_ARG;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(parts_all) || !aligned16(out)) return QSA_ERR_INVALID_ARG;
    return cuda_status(launch_cp_combine(parts_all, n_ranks, (int64_t)n_q * dims->n_q_heads, out, (cudaStream_t)stream));
}

}  // extern "C"
