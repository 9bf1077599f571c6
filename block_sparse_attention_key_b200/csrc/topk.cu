// Exact top-512 block selection over decode score rows (step 3 of the QSA layer).
//
// blog.cecily.jp/6295 (Raschka's explainer paragraph): blocks are taken in
// descending score order, at most 512 of them (2,048 tokens); keieiax.jp glossary
// "Qwen Sparse Attention": 512 blocks per query in the published setting.  The
// pages leave ties open; the lower block index wins here.  The result is a
// compact ascending list per query: no query x key mask exists at any point
// (blog.cecily.jp/6295, first paragraph: the selection is built without kq_mask).
//
// Radix select on 32-bit order-preserving keys.  The first pass (fused into the
// scoring kernel, or k_topk_pass1 here) histograms the top 12 key bits and its
// last CTA fixes the boundary bin b1.  One more pass over the row (k_topk_collect)
// appends every block above b1 to a winner list and every block inside b1 to a
// candidate list; the CTA that finishes that pass last (a completion counter, no
// waiting) settles the selection among the candidates in shared memory (up to 512
// candidates: one sort by key descending and block ascending; more: the remaining
// 20 key bits by radix, then the index tie-break), then sorts the 512 winners.
// When the boundary bin is too crowded (> 4096 candidates, or > 1024 keys equal
// at the cut) the finishing CTA instead re-scans the row in index order.

#include "select_finish.cuh"

namespace qsa {

constexpr int kPerThreadLoad = 16;  // score values each collecting thread holds per sub-chunk

// First histogram pass for score rows that come from the caller (qsa_topk_blocks).
__global__ void __launch_bounds__(256)
k_topk_pass1(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_pos, int32_t row0,
             int64_t kv_capacity, int64_t max_blocks, int bs, int top_k, int chunk, TopkCtrl* __restrict__ ctrl)
{
    __shared__ unsigned s_hist[kBins1];
    __shared__ unsigned s_warp[8];
    __shared__ int s_last;
    griddep_wait();
    griddep_launch_dependents();
    const int tid = threadIdx.x;
    const int r = blockIdx.y;
    TopkCtrl* c = ctrl + r;
    const int64_t n_c = candidate_blocks(q_pos[row0 + r], kv_capacity, max_blocks, bs);
    const int64_t b0 = (int64_t)blockIdx.x * chunk;
    const int64_t b1 = min(b0 + (int64_t)chunk, n_c);
    const float* srow = scores + (int64_t)r * ld;
    for (int k = tid; k < kBins1; k += 256) s_hist[k] = 0;
    __syncthreads();
    for (int64_t b = b0 + tid; b < b1; b += 256) atomicAdd(&s_hist[orderable_key(__ldg(srow + b)) >> 20], 1u);
    __syncthreads();
    for (int k = tid; k < kBins1; k += 256) {
        const unsigned v = s_hist[k];
        if (v) atomicAdd(&c->hist1[k], v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c->done[0], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    finish_digit1(c, n_c, top_k, s_warp);
}

// Collect winners (above the boundary bin) and candidates (inside it); the last
// CTA of a row settles the selection and writes the ascending list.
__global__ void __launch_bounds__(256)
k_topk_collect(const float* __restrict__ scores, int64_t ld, int32_t row0, int chunk, int top_k,
               TopkCtrl* __restrict__ ctrl, unsigned long long* __restrict__ cand, int32_t* __restrict__ tmp,
               int32_t* __restrict__ sel_idx, int32_t* __restrict__ sel_cnt, unsigned* status)
{
    __shared__ FinishSmem S;
    __shared__ int s_base[2];
    __shared__ int s_last;

    griddep_wait();  // everything below reads the scoring pass's results
    griddep_launch_dependents();
    const int tid = threadIdx.x;
    const int r = blockIdx.y;
    const int i = row0 + r;
    TopkCtrl* c = ctrl + r;
    const int64_t n_c = c->n_cand;
    const int mode = c->mode;
    const unsigned b1 = c->prefix;           // top 12 key bits of the boundary bin
    const int need1 = c->need;               // blocks still wanted from that bin
    const bool crowded = c->bin_count > (unsigned)kCandCap;
    const float* srow = scores + (int64_t)r * ld;
    int32_t* win = tmp + (int64_t)r * kSelCap;
    unsigned long long* cl = cand + (int64_t)r * kCandCap;

    if (mode != kSelAll) {
        // sub-chunks of 256 x kPerThreadLoad blocks: every thread loads its values first
        // (independent loads), then one block-wide scan places its winners and candidates
        const int64_t b0 = (int64_t)blockIdx.x * chunk;
        const int64_t b_end = min(b0 + (int64_t)chunk, n_c);
        constexpr int kPer = kPerThreadLoad;
        for (int64_t base = b0; base < b_end; base += 256 * kPer) {
            unsigned key[kPer];
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t b = base + tid + 256 * k;
                key[k] = b < b_end ? orderable_key(__ldg(srow + b)) : 0u;
            }
            unsigned wmask = 0, cmask = 0;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t b = base + tid + 256 * k;
                const unsigned top = key[k] >> 20;
                const bool valid = b < b_end;
                if (valid && (top > b1 || (top == b1 && mode == kSelPrefix))) wmask |= 1u << k;
                if (valid && top == b1 && mode == kSelUndecided && !crowded) cmask |= 1u << k;
            }
            // packed counts: winners in the high 16 bits, candidates in the low 16
            const unsigned mine = ((unsigned)__popc(wmask) << 16) | (unsigned)__popc(cmask);
            unsigned incl = mine;
            const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            if (lane == 31) S.warp[warp] = incl;
            __syncthreads();
            unsigned before = 0, total = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const unsigned v = S.warp[w];
                before += w < warp ? v : 0u;
                total += v;
            }
            if (tid == 0) {
                s_base[0] = (total >> 16) ? (int)atomicAdd(&c->nsel, total >> 16) : 0;
                s_base[1] = (total & 0xFFFFu) ? (int)atomicAdd(&c->ncand, total & 0xFFFFu) : 0;
            }
            __syncthreads();
            const unsigned excl = before + incl - mine;
            int wslot = s_base[0] + (int)(excl >> 16), cslot = s_base[1] + (int)(excl & 0xFFFFu);
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int64_t b = base + tid + 256 * k;
                if (wmask >> k & 1u) {
                    if (wslot < kSelCap) win[wslot] = (int32_t)b;
                    else set_status(status, QSA_DEV_BAD_SEL);
                    ++wslot;
                }
                if (cmask >> k & 1u) {
                    if (cslot < kCandCap) cl[cslot] = ((unsigned long long)key[k] << 32) | (unsigned)b;
                    ++cslot;
                }
            }
            __syncthreads();  // S.warp and s_base are reused by the next sub-chunk
        }
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c->done[1], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int cnt = (int)min((int64_t)top_k, n_c);
    for (int k = tid; k < kSelCap; k += 256) S.list[k] = INT_MAX;
    if (tid == 0) S.n_list = 0;
    __syncthreads();

    bool sorted = false;
    if (mode == kSelAll) {
        for (int k = tid; k < cnt; k += 256) S.list[k] = k;
        sorted = true;
    } else if (mode == kSelPrefix) {
        for (int k = tid; k < cnt; k += 256) S.list[k] = __ldcg(win + k);
    } else if (crowded) {
        select_by_rescan(S, srow, n_c, false, b1, need1);
        sorted = true;
    } else {
        // candidates of the boundary bin, kPerThreadCand per thread, in registers
        const int nc = (int)min(__ldcg(&c->ncand), (unsigned)kCandCap);
        unsigned long long cr[kPerThreadCand];
#pragma unroll
        for (int k = 0; k < kPerThreadCand; ++k) {
            const int j = tid + 256 * k;
            cr[k] = j < nc ? __ldcg(cl + j) : 0ull;
        }
        const int n_win = (int)min(__ldcg(&c->nsel), (unsigned)top_k);
        for (int k = tid; k < n_win; k += 256) S.list[k] = __ldcg(win + k);
        if (tid == 0) S.n_list = n_win;
        __syncthreads();
        if (nc <= kSelCap) {  // a sort of at most kSelCap entries
            // few candidates: sort them by (key desc, block asc) and take the first need1
            take_top_sorted(S, cr, nc, need1);
        } else {
            const Cut cut = resolve_cut_regs(S, cr, nc, need1, false, b1);
            if (!take_by_cut(S, cr, nc, cut)) {
                for (int k = tid; k < kSelCap; k += 256) S.list[k] = INT_MAX;
                __syncthreads();
                select_by_rescan(S, srow, n_c, false, b1, need1);
                sorted = true;
            }
        }
    }
    __syncthreads();
    if (!sorted) sort_list_512(S);
    int32_t* out = sel_idx + (int64_t)i * kSelCap;
    for (int k = tid; k < kSelCap; k += 256) out[k] = k < cnt ? S.list[k] : -1;
    if (tid == 0) sel_cnt[i] = cnt;
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                        int64_t max_blocks, int64_t kv_capacity, int bs, int top_k, int chunk, int n_chunks,
                        TopkCtrl* ctrl,
                        unsigned long long* cand, int32_t* tmp, int32_t* sel_idx, int32_t* sel_cnt, bool hist_done,
                        unsigned* status, cudaStream_t st, bool pdl)
{
    if (n_rows <= 0) return cudaSuccess;
    dim3 grid((unsigned)(n_chunks > 0 ? n_chunks : 1), (unsigned)n_rows);
    if (!hist_done) {
        const cudaError_t e = launch_k(k_topk_pass1, grid, dim3(256), 0, st, false, scores, ld, q_pos, row0,
                                       kv_capacity, max_blocks, bs, top_k, chunk, ctrl);
        if (e != cudaSuccess) return e;
    }
    return launch_k(k_topk_collect, grid, dim3(256), 0, st, hist_done ? pdl : true, scores, ld, row0, chunk, top_k,
                    ctrl, cand, tmp, sel_idx, sel_cnt, status);
}

}  // namespace qsa
