// Exact top-512 block selection over decode score rows (step 3 of the QSA layer).
//
// blog.cecily.jp/6295 (Raschka's explainer paragraph): blocks are taken in
// descending score order, at most 512 of them (2,048 tokens); keieiax.jp glossary
// "Qwen Sparse Attention": 512 blocks per query in the published setting.  The
// pages leave ties open; the lower block index wins here.  The result is a
// compact ascending list per query: no query x key mask exists at any point
// (blog.cecily.jp/6295, first paragraph: the selection is built without kq_mask).
//
// Radix select on 32-bit order-preserving keys, 12 + 12 + 8 bit digits, every
// pass spread over (chunk, row) CTAs so a handful of long rows still fills the
// GPU.  The CTA that finishes a pass last (a completion counter, no waiting)
// fixes the threshold digit; ties on the full key are split by block index using
// per-chunk counts.  The emit pass appends winners to an unordered list and its
// last CTA sorts the <= 512 indices.

#include "select_common.cuh"

namespace qsa {

template <int kLevel>
__global__ void __launch_bounds__(256)
k_topk_pass(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_pos, int32_t row0,
            int64_t kv_capacity, int64_t max_blocks, int chunk, int n_chunks, TopkCtrl* __restrict__ ctrl,
            unsigned* __restrict__ lh3)
{
    constexpr int kBins = kLevel == 3 ? kBins3 : kBins1;
    __shared__ unsigned s_hist[kBins];
    __shared__ unsigned s_warp[8];
    __shared__ int s_last;

    const int tid = threadIdx.x;
    const int r = blockIdx.y;
    TopkCtrl* c = ctrl + r;
    int mode = kSelUndecided;
    unsigned prefix = 0;
    int nbits = 0, need = kTopK;
    if (kLevel > 1) {
        mode = c->mode;
        if (mode != kSelUndecided) return;  // already resolved: nothing to count
        prefix = c->prefix;
        nbits = c->nbits;
        need = c->need;
    }
    // the first pass derives the candidates from the position; later passes reuse the
    // count it recorded (which is 0 for a query the scoring pass rejected)
    const int64_t n_c = kLevel == 1 ? candidate_blocks(q_pos[row0 + r], kv_capacity, max_blocks) : c->n_cand;
    const int64_t b0 = (int64_t)blockIdx.x * chunk;
    const int64_t b1 = min(b0 + (int64_t)chunk, n_c);
    const float* srow = scores + (int64_t)r * ld;

    for (int k = tid; k < kBins; k += 256) s_hist[k] = 0;
    __syncthreads();
    for (int64_t b = b0 + tid; b < b1; b += 256) {
        const unsigned key = orderable_key(__ldg(srow + b));
        if (kLevel == 1) {
            atomicAdd(&s_hist[key >> 20], 1u);
        } else if (kLevel == 2) {
            if ((key >> 20) == prefix) atomicAdd(&s_hist[(key >> 8) & 0xFFFu], 1u);
        } else {
            if ((key >> 8) == prefix) atomicAdd(&s_hist[key & 0xFFu], 1u);
        }
    }
    __syncthreads();
    unsigned* gh = kLevel == 1 ? c->hist1 : (kLevel == 2 ? c->hist2 : c->hist3);
    for (int k = tid; k < kBins; k += 256) {
        const unsigned v = s_hist[k];
        if (kLevel == 3) lh3[((int64_t)r * n_chunks + blockIdx.x) * kBins3 + k] = v;
        if (v) atomicAdd(&gh[k], v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c->done[kLevel - 1], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (kLevel == 1)
        finish_digit1(c, n_c, s_warp);
    else if (kLevel == 2)
        resolve_digit(c, c->hist2, kBins2 / 256, 12, false, prefix, nbits, need, s_warp);
    else
        resolve_digit(c, c->hist3, kBins3 / 256, 8, true, prefix, nbits, need, s_warp);
}

__global__ void __launch_bounds__(256)
k_topk_emit(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_pos, int32_t row0,
            int64_t kv_capacity, int64_t max_blocks, int chunk, int n_chunks, TopkCtrl* __restrict__ ctrl,
            const unsigned* __restrict__ lh3, int32_t* __restrict__ tmp, int32_t* __restrict__ sel_idx,
            int32_t* __restrict__ sel_cnt, unsigned* status)
{
    __shared__ int s_cnt[8];
    __shared__ unsigned s_warp[8];
    __shared__ int s_base;
    __shared__ int s_last;
    __shared__ int s_list[kTopK];

    const int tid = threadIdx.x;
    const int r = blockIdx.y;
    const int i = row0 + r;
    TopkCtrl* c = ctrl + r;
    const int64_t n_c = c->n_cand;
    const int mode = c->mode;
    const unsigned prefix = c->prefix;
    const int nbits = c->nbits;
    const int need = c->need;
    const int shift = 32 - nbits;

    // equal keys in earlier chunks (only needed when ties straddle the cut)
    unsigned eq_before = 0;
    if (mode == kSelTies) {
        unsigned v = 0;
        const unsigned d3 = prefix & 0xFFu;
        for (int cc = tid; cc < (int)blockIdx.x; cc += 256) v += __ldcg(lh3 + ((int64_t)r * n_chunks + cc) * kBins3 + d3);
        eq_before = block_suffix_sum_256(v, s_warp);  // thread 0 holds the total
        if (tid == 0) s_warp[0] = eq_before;
        __syncthreads();
        eq_before = s_warp[0];
        __syncthreads();
    }

    const int64_t b0 = (int64_t)blockIdx.x * chunk;
    const int64_t b1 = min(b0 + (int64_t)chunk, n_c);
    unsigned eq_seen = 0;
    int32_t* out_tmp = tmp + (int64_t)r * kTopK;
    for (int64_t base = b0; base < b1; base += 256) {
        const int64_t b = base + tid;
        const bool valid = b < b1;
        const unsigned key = valid ? orderable_key(__ldg(scores + (int64_t)r * ld + b)) : 0u;
        bool take;
        if (mode == kSelAll) {
            take = valid;
        } else if (mode == kSelPrefix) {
            take = valid && (key >> shift) >= prefix;
        } else {  // kSelTies: prefix is the full threshold key
            const bool eq = valid && key == prefix;
            int eq_total;
            const int eq_rank = block_rank_256(eq, s_cnt, &eq_total);
            take = (valid && key > prefix) || (eq && (int)(eq_before + eq_seen) + eq_rank < need);
            eq_seen += (unsigned)eq_total;
        }
        int n_take;
        const int rank = block_rank_256(take, s_cnt, &n_take);
        if (n_take == 0) continue;
        if (tid == 0) s_base = (int)atomicAdd(&c->nsel, (unsigned)n_take);
        __syncthreads();
        if (take) {
            const int slot = s_base + rank;
            if (slot < kTopK) out_tmp[slot] = (int32_t)b;
            else set_status(status, QSA_DEV_BAD_SEL);
        }
        __syncthreads();
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c->done[3], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int cnt = (int)min((int64_t)kTopK, n_c);
    for (int k = tid; k < kTopK; k += 256) s_list[k] = k < cnt ? __ldcg(out_tmp + k) : 0;
    __syncthreads();
    int32_t* out = sel_idx + (int64_t)i * kTopK;
    for (int k = tid; k < kTopK; k += 256) {
        if (k < cnt) {
            const int v = s_list[k];
            int rank = 0;
            for (int j = 0; j < cnt; ++j) rank += s_list[j] < v;
            out[rank] = v;
        } else {
            out[k] = -1;
        }
    }
    if (tid == 0) sel_cnt[i] = cnt;
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                        int64_t max_blocks, int64_t kv_capacity, int chunk, int n_chunks, TopkCtrl* ctrl,
                        unsigned* lh3, int32_t* tmp, int32_t* sel_idx, int32_t* sel_cnt, bool hist_done,
                        unsigned* status, cudaStream_t st)
{
    if (n_rows <= 0) return cudaSuccess;
    dim3 grid((unsigned)(n_chunks > 0 ? n_chunks : 1), (unsigned)n_rows);
    if (!hist_done)
        k_topk_pass<1><<<grid, 256, 0, st>>>(scores, ld, q_pos, row0, kv_capacity, max_blocks, chunk,
                                             n_chunks, ctrl, lh3);
    k_topk_pass<2><<<grid, 256, 0, st>>>(scores, ld, q_pos, row0, kv_capacity, max_blocks, chunk, n_chunks,
                                         ctrl, lh3);
    k_topk_pass<3><<<grid, 256, 0, st>>>(scores, ld, q_pos, row0, kv_capacity, max_blocks, chunk, n_chunks,
                                         ctrl, lh3);
    k_topk_emit<<<grid, 256, 0, st>>>(scores, ld, q_pos, row0, kv_capacity, max_blocks, chunk, n_chunks, ctrl,
                                      lh3, tmp, sel_idx, sel_cnt, status);
    return cudaGetLastError();
}

}  // namespace qsa
