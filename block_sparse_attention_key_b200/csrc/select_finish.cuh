// Block-level (256 threads) exact top-k finishers shared by the decode select
// and the prefill select.  Keys are 32-bit order-preserving encodings of fp32
// scores; the top `need` are taken by (key descending, block index ascending).
// Radix digits: bits 31..20 (4096 bins), 19..8 (4096 bins), 7..0 (256 bins).
#pragma once

#include <climits>

#include "select_common.cuh"

namespace qsa {

constexpr int kPerThreadCand = kCandCap / 256;  // candidates each finishing thread holds
constexpr int kMaxTieRank = 1024;               // keys equal at the cut ranked pairwise at most

struct FinishSmem {
    unsigned hist[kBins2];
    int list[kTopK];
    unsigned warp[8];
    int cnt[8];
    int n_list;
    unsigned res_digit, res_count;
    int res_need;
    int neq;
};

// Among candidates counted in S.hist[0 .. 256*kPer) find the digit holding the
// need-th largest: S.res_digit, S.res_need (still wanted inside it), S.res_count.
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

__device__ __forceinline__ void clear_hist(FinishSmem& S, int nbins)
{
    for (int k = threadIdx.x; k < nbins; k += 256) S.hist[k] = 0;
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

// The cut of a selection: keys > cut are taken; keys == cut are all taken when
// `whole`, else only the `need` with the lowest block indices.
struct Cut {
    unsigned key;
    int need;
    bool whole;
};

// Resolve the cut among candidates held in registers (kPerThreadCand per thread,
// entry = key << 32 | block, `nc` valid in total).  If `from_digit1` is false all
// candidates share the top 12 bits `p12`.  `need` >= 1 candidates are wanted.
__device__ __forceinline__ Cut resolve_cut_regs(FinishSmem& S, const unsigned long long (&cr)[kPerThreadCand],
                                                int nc, int need, bool from_digit1, unsigned p12)
{
    const int tid = threadIdx.x;
    if (from_digit1) {
        clear_hist(S, kBins1);
#pragma unroll
        for (int k = 0; k < kPerThreadCand; ++k)
            if (tid + 256 * k < nc) atomicAdd(&S.hist[(unsigned)(cr[k] >> 52)], 1u);
        __syncthreads();
        resolve_smem<kBins1 / 256>(S, need);
        p12 = S.res_digit;
        need = S.res_need;
        if (S.res_count == (unsigned)need) {
            __syncthreads();
            return Cut{p12 << 20, need, true};
        }
        __syncthreads();
    }
    clear_hist(S, kBins2);
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        if (tid + 256 * k < nc && (unsigned)(cr[k] >> 52) == p12) atomicAdd(&S.hist[(unsigned)(cr[k] >> 40) & 0xFFFu], 1u);
    __syncthreads();
    resolve_smem<kBins2 / 256>(S, need);
    const unsigned p24 = (p12 << 12) | S.res_digit;
    need = S.res_need;
    if (S.res_count == (unsigned)need) {
        __syncthreads();
        return Cut{p24 << 8, need, true};
    }
    __syncthreads();
    clear_hist(S, kBins3);
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k)
        if (tid + 256 * k < nc && (unsigned)(cr[k] >> 40) == p24) atomicAdd(&S.hist[(unsigned)(cr[k] >> 32) & 0xFFu], 1u);
    __syncthreads();
    resolve_smem<1>(S, need);
    const Cut c{(p24 << 8) | S.res_digit, S.res_need, S.res_count == (unsigned)S.res_need};
    S.neq = (int)S.res_count;
    __syncthreads();
    return c;
}

// Append the candidates taken by `c` to S.list (after S.n_list existing entries).
// Returns false when too many keys tie at the cut to rank them pairwise.
__device__ __forceinline__ bool take_by_cut(FinishSmem& S, const unsigned long long (&cr)[kPerThreadCand], int nc,
                                            const Cut& c)
{
    const int tid = threadIdx.x;
    if (!c.whole && S.neq > kMaxTieRank) return false;
    int* eq_idx = reinterpret_cast<int*>(S.hist);  // block indices of keys equal to the cut
    __shared__ int s_neq;
    if (tid == 0) s_neq = 0;
    __syncthreads();
    if (!c.whole) {
#pragma unroll
        for (int k = 0; k < kPerThreadCand; ++k)
            if (tid + 256 * k < nc && (unsigned)(cr[k] >> 32) == c.key) eq_idx[atomicAdd(&s_neq, 1)] = (int)(unsigned)cr[k];
    }
    __syncthreads();
    const int neq = s_neq;
#pragma unroll
    for (int k = 0; k < kPerThreadCand; ++k) {
        if (tid + 256 * k >= nc) continue;
        const unsigned key = (unsigned)(cr[k] >> 32);
        const int b = (int)(unsigned)cr[k];
        bool take = key > c.key || (key == c.key && c.whole);
        if (!take && key == c.key) {
            int rank = 0;
            for (int j = 0; j < neq; ++j) rank += eq_idx[j] < b;
            take = rank < c.need;
        }
        if (take) {
            const int slot = atomicAdd(&S.n_list, 1);
            if (slot < kTopK) S.list[slot] = b;
        }
    }
    __syncthreads();
    return true;
}

// Ordered selection of the top `need` keys of a score row in global memory
// (keys whose top 12 bits exceed `p12` are all taken; among those equal to it the
// top `need12`), written to S.list in ascending block order.  With `from_digit1`
// the whole row is ranked (p12 and need12 are ignored; need12 = top_k).
__device__ inline void select_by_rescan(FinishSmem& S, const float* srow, int64_t n_c, bool from_digit1, unsigned p12,
                                 int need12)
{
    const int tid = threadIdx.x;
    int need = need12;
    unsigned cut;
    bool whole = false;
    if (from_digit1) {
        need = kTopK;
        clear_hist(S, kBins1);
        for (int64_t b = tid; b < n_c; b += 256) atomicAdd(&S.hist[orderable_key(__ldcg(srow + b)) >> 20], 1u);
        __syncthreads();
        resolve_smem<kBins1 / 256>(S, need);
        p12 = S.res_digit;
        need = S.res_need;
        whole = S.res_count == (unsigned)need;
        __syncthreads();
    }
    cut = p12 << 20;
    if (!whole) {
        clear_hist(S, kBins2);
        for (int64_t b = tid; b < n_c; b += 256) {
            const unsigned key = orderable_key(__ldcg(srow + b));
            if ((key >> 20) == p12) atomicAdd(&S.hist[(key >> 8) & 0xFFFu], 1u);
        }
        __syncthreads();
        resolve_smem<kBins2 / 256>(S, need);
        const unsigned p24 = (p12 << 12) | S.res_digit;
        need = S.res_need;
        cut = p24 << 8;
        whole = S.res_count == (unsigned)need;
        __syncthreads();
        if (!whole) {
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
            __syncthreads();
        }
    }
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

}  // namespace qsa
