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
// waiting) settles the remaining 20 key bits and the index tie-break among the
// candidates in registers and shared memory, then bitonic-sorts the 512 winners.
// When the boundary bin is too crowded (>= 4096 candidates, or > 1024 keys equal
// at the cut) the finishing CTA instead re-scans the row in index order.

#include "select_common.cuh"

namespace qsa {

namespace {

constexpr int kPerThreadCand = kCandCap / 256;  // candidates each finishing thread holds
constexpr int kMaxTieRank = 1024;               // equal keys ranked pairwise at most

struct FinishSmem {
    unsigned hist[kBins2];
    int list[kTopK];
    unsigned warp[8];
    int cnt[8];
    int n_list;
    unsigned res_digit, res_count;
    int res_need;
};

// Smem twin of resolve_digit: among candidates counted in hist[0 .. 256*kPer),
// find the digit holding the need-th largest; returns (digit, need left in it, bin count).
template <int kPer>
__device__ __forceinline__ void resolve_smem(FinishSmem& S, int need)
{
    const int tid = threadIdx.x;
    unsigned h[kPer];
    unsigned local = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        h[k] = S.hist[tid * kPer + k];
        local += h[k];
    }
    const unsigned suf = block_suffix_sum_256(local, S.warp);
    const unsigned after = suf - local;
    if (suf >= (unsigned)need && after < (unsigned)need) {
        unsigned run = after;
        int found = -1;
        unsigned fh = 0, frun = 0;
#pragma unroll
        for (int k = kPer - 1; k >= 0; --k) {
            if (found < 0 && run + h[k] >= (unsigned)need) {
                found = k;
                fh = h[k];
                frun = run;
            }
            run += h[k];
        }
        S.res_digit = (unsigned)(tid * kPer + found);
        S.res_count = fh;
        S.res_need = need - (int)frun;
    }
    __syncthreads();
}

// Ascending bitonic sort of S.list[0..512) (unused slots hold INT_MAX).
__device__ __forceinline__ void bitonic_sort_512(FinishSmem& S)
{
    const int tid = threadIdx.x;
    for (int k = 2; k <= kTopK; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int i = (tid / j) * 2 * j + (tid % j);
            const int l = i + j;
            const int a = S.list[i], b = S.list[l];
            const bool up = (i & k) == 0;
            if ((a > b) == up) {
                S.list[i] = b;
                S.list[l] = a;
            }
            __syncthreads();
        }
    }
}

__device__ __forceinline__ void clear_hist(FinishSmem& S, int nbins)
{
    for (int k = threadIdx.x; k < nbins; k += 256) S.hist[k] = 0;
    __syncthreads();
}

// Ordered single-CTA selection from the global score row, for crowded boundaries.
// Keys above the cut are taken; keys equal to it are taken in block order.
__device__ void finish_by_rescan(FinishSmem& S, const float* srow, int64_t n_c, unsigned b1, int need1)
{
    const int tid = threadIdx.x;
    // digit 2 among keys in bin b1
    clear_hist(S, kBins2);
    for (int64_t b = tid; b < n_c; b += 256) {
        const unsigned key = orderable_key(__ldcg(srow + b));
        if ((key >> 20) == b1) atomicAdd(&S.hist[(key >> 8) & 0xFFFu], 1u);
    }
    __syncthreads();
    resolve_smem<kBins2 / 256>(S, need1);
    const unsigned p24 = (b1 << 12) | S.res_digit;
    int need = S.res_need;
    unsigned cut = p24 << 8;  // smallest key taken
    bool whole = S.res_count == (unsigned)need;
    if (!whole) {
        __syncthreads();
        clear_hist(S, kBins3);
        for (int64_t b = tid; b < n_c; b += 256) {
            const unsigned key = orderable_key(__ldcg(srow + b));
            if ((key >> 8) == p24) atomicAdd(&S.hist[key & 0xFFu], 1u);
        }
        __syncthreads();
        resolve_smem<1>(S, need);
        cut = (p24 << 8) | S.res_digit;
        need = S.res_need;
        whole = S.res_count == (unsigned)need;
    }
    // keys >= cut are taken, except that among keys == cut only the first `need` (when not whole)
    int taken = 0, eq_seen = 0;
    for (int64_t base = 0; base < n_c; base += 256) {
        const int64_t b = base + tid;
        const bool valid = b < n_c;
        const unsigned key = valid ? orderable_key(__ldcg(srow + b)) : 0u;
        int eq_total;
        const bool eq = valid && key == cut;
        const int eq_rank = block_rank_256(eq, S.cnt, &eq_total);
        const bool take = valid && (key > cut || (eq && (whole || eq_seen + eq_rank < need)));
        int n_take;
        const int rank = block_rank_256(take, S.cnt, &n_take);
        if (take && taken + rank < kTopK) S.list[taken + rank] = (int)b;
        taken += n_take;
        eq_seen += eq_total;
    }
    __syncthreads();
    if (tid == 0) S.n_list = taken < kTopK ? taken : kTopK;
    __syncthreads();
}

}  // namespace

// First histogram pass for score rows that come from the caller (qsa_topk_blocks).
__global__ void __launch_bounds__(256)
k_topk_pass1(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_pos, int32_t row0,
             int64_t kv_capacity, int64_t max_blocks, int chunk, TopkCtrl* __restrict__ ctrl)
{
    __shared__ unsigned s_hist[kBins1];
    __shared__ unsigned s_warp[8];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    const int r = blockIdx.y;
    TopkCtrl* c = ctrl + r;
    const int64_t n_c = candidate_blocks(q_pos[row0 + r], kv_capacity, max_blocks);
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
    finish_digit1(c, n_c, s_warp);
}

// Collect winners (above the boundary bin) and candidates (inside it); the last
// CTA of a row settles the selection and writes the ascending list.
__global__ void __launch_bounds__(256)
k_topk_collect(const float* __restrict__ scores, int64_t ld, int32_t row0, int chunk, TopkCtrl* __restrict__ ctrl,
               unsigned long long* __restrict__ cand, int32_t* __restrict__ tmp, int32_t* __restrict__ sel_idx,
               int32_t* __restrict__ sel_cnt, unsigned* status)
{
    __shared__ FinishSmem S;
    __shared__ int s_base[2];
    __shared__ int s_last;

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
    int32_t* win = tmp + (int64_t)r * kTopK;
    unsigned long long* cl = cand + (int64_t)r * kCandCap;

    if (mode != kSelAll) {
        const int64_t b0 = (int64_t)blockIdx.x * chunk;
        const int64_t b_end = min(b0 + (int64_t)chunk, n_c);
        for (int64_t base = b0; base < b_end; base += 256) {
            const int64_t b = base + tid;
            const bool valid = b < b_end;
            const unsigned key = valid ? orderable_key(__ldg(srow + b)) : 0u;
            const unsigned top = key >> 20;
            const bool is_win = valid && (top > b1 || (top == b1 && mode == kSelPrefix));
            const bool is_cand = valid && top == b1 && mode == kSelUndecided && !crowded;
            int n_win, n_cand;
            const int rw = block_rank_256(is_win, S.cnt, &n_win);
            const int rc = block_rank_256(is_cand, S.cnt, &n_cand);
            if (n_win == 0 && n_cand == 0) continue;
            if (tid == 0) {
                s_base[0] = n_win ? (int)atomicAdd(&c->nsel, (unsigned)n_win) : 0;
                s_base[1] = n_cand ? (int)atomicAdd(&c->ncand, (unsigned)n_cand) : 0;
            }
            __syncthreads();
            if (is_win) {
                const int slot = s_base[0] + rw;
                if (slot < kTopK) win[slot] = (int32_t)b;
                else set_status(status, QSA_DEV_BAD_SEL);
            }
            if (is_cand) {
                const int slot = s_base[1] + rc;
                if (slot < kCandCap) cl[slot] = ((unsigned long long)key << 32) | (unsigned)b;
            }
            __syncthreads();
        }
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&c->done[1], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int cnt = (int)min((int64_t)kTopK, n_c);
    for (int k = tid; k < kTopK; k += 256) S.list[k] = INT_MAX;
    if (tid == 0) S.n_list = 0;
    __syncthreads();

    bool sorted = false;
    if (mode == kSelAll) {
        for (int k = tid; k < cnt; k += 256) S.list[k] = k;
        sorted = true;
    } else if (mode == kSelPrefix) {
        for (int k = tid; k < kTopK; k += 256) S.list[k] = __ldcg(win + k);
    } else if (crowded) {
        finish_by_rescan(S, srow, n_c, b1, need1);
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
        // digit 2: key bits 19..8
        clear_hist(S, kBins2);
#pragma unroll
        for (int k = 0; k < kPerThreadCand; ++k)
            if (tid + 256 * k < nc) atomicAdd(&S.hist[(unsigned)(cr[k] >> 40) & 0xFFFu], 1u);
        __syncthreads();
        resolve_smem<kBins2 / 256>(S, need1);
        const unsigned p24 = (b1 << 12) | S.res_digit;
        int need = S.res_need;
        unsigned cut = p24 << 8;
        bool whole = S.res_count == (unsigned)need;
        unsigned eq_count = 0;
        if (!whole) {
            __syncthreads();
            clear_hist(S, kBins3);
#pragma unroll
            for (int k = 0; k < kPerThreadCand; ++k)
                if (tid + 256 * k < nc && (unsigned)(cr[k] >> 40) == p24)
                    atomicAdd(&S.hist[(unsigned)(cr[k] >> 32) & 0xFFu], 1u);
            __syncthreads();
            resolve_smem<1>(S, need);
            cut = (p24 << 8) | S.res_digit;
            need = S.res_need;
            eq_count = S.res_count;
            whole = eq_count == (unsigned)need;
        }
        if (!whole && eq_count > (unsigned)kMaxTieRank) {
            __syncthreads();
            finish_by_rescan(S, srow, n_c, b1, need1);
            sorted = true;
        } else {
            // winners first, then the chosen candidates
            const int n_win = (int)min(__ldcg(&c->nsel), (unsigned)kTopK);
            for (int k = tid; k < n_win; k += 256) S.list[k] = __ldcg(win + k);
            if (tid == 0) S.n_list = n_win;
            // block indices of the keys equal to the cut, for the index tie-break
            int* eq_idx = reinterpret_cast<int*>(S.hist);
            __shared__ int s_neq;
            if (tid == 0) s_neq = 0;
            __syncthreads();
            if (!whole) {
#pragma unroll
                for (int k = 0; k < kPerThreadCand; ++k)
                    if (tid + 256 * k < nc && (unsigned)(cr[k] >> 32) == cut)
                        eq_idx[atomicAdd(&s_neq, 1)] = (int)(unsigned)cr[k];
            }
            __syncthreads();
            const int neq = s_neq;
#pragma unroll
            for (int k = 0; k < kPerThreadCand; ++k) {
                if (tid + 256 * k >= nc) continue;
                const unsigned key = (unsigned)(cr[k] >> 32);
                const int b = (int)(unsigned)cr[k];
                bool take = key > cut || (key == cut && whole);
                if (!take && key == cut) {
                    int rank = 0;
                    for (int j = 0; j < neq; ++j) rank += eq_idx[j] < b;
                    take = rank < need;
                }
                if (take) {
                    const int slot = atomicAdd(&S.n_list, 1);
                    if (slot < kTopK) S.list[slot] = b;
                }
            }
            __syncthreads();
        }
    }
    __syncthreads();
    if (!sorted) bitonic_sort_512(S);
    int32_t* out = sel_idx + (int64_t)i * kTopK;
    for (int k = tid; k < kTopK; k += 256) out[k] = k < cnt ? S.list[k] : -1;
    if (tid == 0) sel_cnt[i] = cnt;
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int32_t row0, int32_t n_rows,
                        int64_t max_blocks, int64_t kv_capacity, int chunk, int n_chunks, TopkCtrl* ctrl,
                        unsigned long long* cand, int32_t* tmp, int32_t* sel_idx, int32_t* sel_cnt, bool hist_done,
                        unsigned* status, cudaStream_t st)
{
    if (n_rows <= 0) return cudaSuccess;
    dim3 grid((unsigned)(n_chunks > 0 ? n_chunks : 1), (unsigned)n_rows);
    if (!hist_done)
        k_topk_pass1<<<grid, 256, 0, st>>>(scores, ld, q_pos, row0, kv_capacity, max_blocks, chunk, ctrl);
    k_topk_collect<<<grid, 256, 0, st>>>(scores, ld, row0, chunk, ctrl, cand, tmp, sel_idx, sel_cnt, status);
    return cudaGetLastError();
}

}  // namespace qsa
