// Device helpers of the exact top-k block selection (256-thread CTAs).
//
// The selection keeps, per query, the top_k candidates by (score descending,
// block index ascending).  It is a radix select on 32-bit order-preserving keys
// of the fp32 scores: digit 1 = key bits 31..20, digit 2 = bits 19..8,
// digit 3 = bits 7..0.  After each digit's histogram the CTA that finishes last
// fixes that digit of the threshold key; ties on the full key are then broken by
// block index using per-chunk counts (chunks are in index order).
#pragma once

#include "qsa_internal.cuh"

namespace qsa {

// Inclusive suffix sum over the 256 threads of the CTA: returns sum_{t >= tid} v[t].
__device__ __forceinline__ unsigned block_suffix_sum_256(unsigned v, unsigned* s_warp /*[8]*/)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_down_sync(0xffffffffu, v, off);
        if (lane + off < 32) v += o;
    }
    if (lane == 0) s_warp[warp] = v;  // warp total
    __syncthreads();
    unsigned later = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w)
        if (w > warp) later += s_warp[w];
    __syncthreads();
    return v + later;
}

// Exclusive prefix count of a predicate over the 256 threads, in thread order.
// Returns this thread's rank among the true predicates; *total gets the count.
__device__ __forceinline__ int block_rank_256(bool p, int* s_cnt /*[8]*/, int* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned m = __ballot_sync(0xffffffffu, p);
    if (lane == 0) s_cnt[warp] = __popc(m);
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const int c = s_cnt[w];
        before += (w < warp) ? c : 0;
        all += c;
    }
    __syncthreads();
    *total = all;
    return before + __popc(m & ((1u << lane) - 1u));
}

// Fix the next digit of the threshold key.  Run by all 256 threads of the CTA
// that completed a histogram pass.  `hist` (global, 256 * kPer bins) counts the
// candidates whose key matches the resolved prefix, by their next digit.  Among
// them the top `need` are wanted.  Updates ctrl->{prefix, nbits, need, mode}.
// Each thread owns kPer consecutive bins, loaded once (independent loads).
template <int kPer>
__device__ __forceinline__ void resolve_digit(TopkCtrl* ctrl, const unsigned* hist, int bits, bool final_digit,
                                              unsigned prefix, int nbits, int need, unsigned* s_warp)
{
    const int tid = threadIdx.x;
    unsigned h[kPer];
    unsigned local = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) h[k] = __ldcg(hist + tid * kPer + k);
#pragma unroll
    for (int k = 0; k < kPer; ++k) local += h[k];
    const unsigned suf = block_suffix_sum_256(local, s_warp);
    const unsigned after = suf - local;
    if (suf >= (unsigned)need && after < (unsigned)need) {
        unsigned run = after;
        int found = -1;
        unsigned found_h = 0, found_run = 0;
#pragma unroll
        for (int k = kPer - 1; k >= 0; --k) {
            if (found < 0 && run + h[k] >= (unsigned)need) {
                found = k;
                found_h = h[k];
                found_run = run;
            }
            run += h[k];
        }
        const unsigned digit = (unsigned)(tid * kPer + found);
        const int need_here = need - (int)found_run;
        ctrl->prefix = (prefix << bits) | digit;
        ctrl->nbits = nbits + bits;
        ctrl->need = need_here;
        ctrl->bin_count = found_h;
        ctrl->mode = (found_h == (unsigned)need_here) ? kSelPrefix : (final_digit ? kSelTies : kSelUndecided);
    }
}

// Candidates of query row: n_c(t) = floor((t+1)/bs), cut at max_blocks; 0 for an invalid position.
__device__ __forceinline__ int64_t candidate_blocks(int t, int64_t kv_capacity, int64_t max_blocks, int bs)
{
    if (t < 0 || (int64_t)t >= kv_capacity) return 0;
    const int64_t n_c = ((int64_t)t + 1) / bs;
    return n_c < max_blocks ? n_c : max_blocks;
}

// Completion of digit 1 (run by the last CTA of the first histogram pass).
__device__ __forceinline__ void finish_digit1(TopkCtrl* ctrl, int64_t n_c, int top_k, unsigned* s_warp)
{
    if (n_c <= top_k) {
        if (threadIdx.x == 0) {
            ctrl->n_cand = (int)n_c;
            ctrl->mode = kSelAll;
        }
        return;
    }
    if (threadIdx.x == 0) ctrl->n_cand = (int)n_c;
    resolve_digit<kBins1 / 256>(ctrl, ctrl->hist1, 12, false, 0u, 0, top_k, s_warp);
}

}  // namespace qsa
