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
    if (d->block_size != kBlock || d->top_k != kTopK) return QSA_ERR_INVALID_ARG;
    if (d->kv_capacity <= 0 || d->kv_capacity % kBlock != 0 || d->kv_capacity >= (1ll << 31))
        return QSA_ERR_INVALID_ARG;
    if (!std::isfinite(d->softmax_scale)) return QSA_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim || d->n_idx_heads != kIdxHeads || d->idx_dim != kIdxDim)
        return QSA_ERR_UNSUPPORTED;
    if (d->n_q_heads / d->n_kv_heads > kMaxGroup) return QSA_ERR_UNSUPPORTED;
    return QSA_OK;
}

int check_rows(const qsa_dims* d, int32_t n_q, int64_t max_blocks)
{
    if (n_q < 0 || max_blocks < 0 || max_blocks > d->kv_capacity / kBlock) return QSA_ERR_INVALID_ARG;
    if (n_q > 65535) return QSA_ERR_UNSUPPORTED;
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
    L.n_split = mode == QSA_MODE_PREFILL ? 1 : attn_splits(n_q, d.n_kv_heads);

    // zeroed region: attention split counters, then the select control blocks
    L.attn_cnt = off;
    L.ctrl = off + align_up((size_t)n_q * d.n_kv_heads * 4);
    L.ctrl_bytes = (L.ctrl - L.attn_cnt) + (size_t)rows * sizeof(TopkCtrl);
    off = L.attn_cnt + align_up(L.ctrl_bytes);
    L.cand = off;
    off += align_up((size_t)rows * kCandCap * 8);
    L.tmp = off;
    off += align_up((size_t)rows * kTopK * 4);
    L.score_ld = (max_blocks + 3) / 4 * 4;
    L.scores = off;
    off += align_up((size_t)rows * L.score_ld * 4);
    L.sel = off;
    off += align_up((size_t)n_q * kTopK * 4 + (size_t)n_q * 4);
    L.partial = off;
    if (L.n_split > 1) off += align_up((size_t)n_q * d.n_kv_heads * L.n_split * (32 + 16 * kHeadDim) * 4);
    if (mode == QSA_MODE_PREFILL && max_blocks > 0 && n_q > 0) {
        L.pf_split = prefill_splits(n_q, max_blocks);
        const size_t segs = (size_t)n_q * 2 * L.pf_split;
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
    L.total = off;
    return L;
}

}  // namespace qsa

using namespace qsa;

extern "C" {

size_t qsa_workspace_bytes(const qsa_dims* dims, int32_t n_q, int64_t max_blocks, int32_t mode)
{
    if (check_dims(dims) != QSA_OK || check_rows(dims, n_q, max_blocks) != QSA_OK) return 0;
    if (mode != QSA_MODE_DECODE && mode != QSA_MODE_PREFILL) return 0;
    return plan_workspace(*dims, n_q, max_blocks, mode).total;
}

int qsa_workspace_init(void* workspace, size_t ws_bytes, void* stream)
{
    if (!aligned16(workspace) || ws_bytes < kAlign) return QSA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(workspace, 0, kAlign, (cudaStream_t)stream));
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
        cudaError_t e = cudaMemsetAsync(sel_idx, 0xFF, (size_t)n_q * kTopK * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(sel_cnt, 0, (size_t)n_q * 4, st);
        return cuda_status(e);
    }
    cudaError_t e = cudaMemsetAsync(ws + L.attn_cnt, 0, L.ctrl_bytes, st);
    if (e != cudaSuccess) return QSA_ERR_CUDA;
    return cuda_status(launch_topk(scores, ld_scores, q_pos, 0, n_q, max_blocks, dims->kv_capacity, L.chunk,
                                   L.n_chunks, (TopkCtrl*)(ws + L.ctrl), (unsigned long long*)(ws + L.cand),
                                   (int32_t*)(ws + L.tmp), sel_idx, sel_cnt, false, (unsigned*)ws, st));
}

int qsa_sparse_attn(const qsa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel_idx, const int32_t* sel_cnt,
                    int32_t n_q, void* out, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if ((rc = check_rows(dims, n_q, 0)) != QSA_OK) return rc;
    if (n_q == 0) return QSA_OK;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q_seq) || !aligned16(q_pos) ||
        !aligned16(sel_idx) || !aligned16(sel_cnt) || !aligned16(out) || !aligned16(workspace))
        return QSA_ERR_INVALID_ARG;
    const WsLayout L = plan_workspace(*dims, n_q, 0, QSA_MODE_DECODE);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    if (L.n_split > 1) {
        cudaError_t e = cudaMemsetAsync(ws + L.attn_cnt, 0, (size_t)n_q * dims->n_kv_heads * 4, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    return cuda_status(launch_attention(*dims, q, k_cache, v_cache, q_seq, q_pos, sel_idx, sel_cnt, n_q, out,
                                        L.n_split, (float*)(ws + L.partial), (unsigned*)(ws + L.attn_cnt),
                                        (unsigned*)ws, st));
}

int qsa_forward(const qsa_dims* dims, const qsa_forward_args* a, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_dims(dims);
    if (rc != QSA_OK) return rc;
    if (!a) return QSA_ERR_INVALID_ARG;
    if ((rc = check_rows(dims, a->n_q, a->max_blocks)) != QSA_OK) return rc;
    if (a->mode != QSA_MODE_DECODE && a->mode != QSA_MODE_PREFILL) return QSA_ERR_INVALID_ARG;
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
    const WsLayout L = plan_workspace(*dims, n_q, a->max_blocks, a->mode);
    if (ws_bytes < L.total) return QSA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t st = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    unsigned* status = (unsigned*)ws;
    cudaError_t e = cudaSuccess;
    int32_t* sel_idx = a->sel_idx ? a->sel_idx : (int32_t*)(ws + L.sel);
    int32_t* sel_cnt = a->sel_cnt ? a->sel_cnt : (int32_t*)(ws + L.sel) + (size_t)n_q * kTopK;

    if (n_q > 0 && a->max_blocks > 0 && a->mode == QSA_MODE_DECODE) {
        // decode chain, each kernel launched as a programmatic dependent of the one
        // before: pool (+ clearing of the split counters and select control blocks),
        // scores with the digit-1 histogram, select, attention
        e = launch_pool(*dims, a->idx_k, a->pooled, a->len_before, a->len_after, a->max_new_tokens, ws + L.attn_cnt,
                        L.ctrl_bytes, status, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
        TopkCtrl* ctrl = (TopkCtrl*)(ws + L.ctrl);
        float* scores = (float*)(ws + L.scores);
        // rows of up to 16,384 blocks are selected by the scoring kernel's last CTA per row
        const bool in_kernel = a->max_blocks <= kScoreFinishMaxBlocks;
        e = launch_score_decode(*dims, a->q_idx, a->w, a->pooled, a->q_seq, a->q_pos, 0, n_q, a->max_blocks, scores,
                                L.score_ld, L.chunk, ctrl, in_kernel ? sel_idx : nullptr,
                                in_kernel ? sel_cnt : nullptr, status, st, true);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
        if (!in_kernel) {
            e = launch_topk(scores, L.score_ld, a->q_pos, 0, n_q, a->max_blocks, dims->kv_capacity, L.chunk,
                            L.n_chunks, ctrl, (unsigned long long*)(ws + L.cand), (int32_t*)(ws + L.tmp), sel_idx,
                            sel_cnt, true, status, st, true);
            if (e != cudaSuccess) return QSA_ERR_CUDA;
        }
        return cuda_status(launch_attention(*dims, a->q, a->k_cache, a->v_cache, a->q_seq, a->q_pos, sel_idx,
                                            sel_cnt, n_q, a->out, L.n_split, (float*)(ws + L.partial),
                                            (unsigned*)(ws + L.attn_cnt), status, st, true));
    }

    if (a->max_new_tokens > 0) {
        e = launch_pool(*dims, a->idx_k, a->pooled, a->len_before, a->len_after, a->max_new_tokens, nullptr, 0,
                        status, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    if (n_q == 0) return QSA_OK;

    if (a->max_blocks == 0) {
        e = cudaMemsetAsync(sel_idx, 0xFF, (size_t)n_q * kTopK * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(sel_cnt, 0, (size_t)n_q * 4, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    } else {
        // prefill chunk: tensor-core scoring with streaming admission
        e = cudaMemsetAsync(ws + L.pf_theta, 0, (size_t)(n_q + 1) * 4, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
        e = launch_prefill_select(*dims, a->q_idx, a->w, a->pooled, a->q_seq, a->q_pos, n_q, a->max_blocks,
                                  L.pf_split, (unsigned long long*)(ws + L.pf_cand), (unsigned*)(ws + L.pf_cnt),
                                  (unsigned*)(ws + L.pf_theta), (uint32_t*)(ws + L.pf_shist), (int32_t*)(ws + L.pf_work),
                                  (float*)(ws + L.pf_scratch), L.pf_fb_ctas, sel_idx, sel_cnt, status, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    if (L.n_split > 1) {
        e = cudaMemsetAsync(ws + L.attn_cnt, 0, (size_t)n_q * dims->n_kv_heads * 4, st);
        if (e != cudaSuccess) return QSA_ERR_CUDA;
    }
    return cuda_status(launch_attention(*dims, a->q, a->k_cache, a->v_cache, a->q_seq, a->q_pos, sel_idx, sel_cnt,
                                        n_q, a->out, L.n_split, (float*)(ws + L.partial),
                                        (unsigned*)(ws + L.attn_cnt), status, st));
}

}  // extern "C"
